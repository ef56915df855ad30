// C ABI of libttt_b200: argument validation and dispatch (see include/ttt.h).
#include <mutex>

#include "common.cuh"
#include "lact.cuh"

namespace {

__device__ int g_device_status;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;

// Device address of the status word on the current device (looked up once
// per device; the symbol itself is a host-side handle, not an address).
int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

size_t elem_size(int32_t dtype) { return dtype == TTT_BF16 ? 2 : 4; }

// Sizes the kernels index with 32-bit integers: tokens per sequence (tile
// starts plus one tile stay below 2^31) and (batch, head) pairs (grids of a
// few CTAs per pair).
constexpr int64_t kMaxT = (int64_t)1 << 30;
constexpr int64_t kMaxHeads = (int64_t)1 << 24;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte range [lo, hi) touched by a strided tensor (non-negative strides).
struct Extent {
  uintptr_t lo, hi;
};
Extent extent(const ttt_tensor* t) {
  uintptr_t base = reinterpret_cast<uintptr_t>(t->data);
  int64_t last = 0;
  for (int i = 0; i < t->ndim; ++i) last += (t->shape[i] - 1) * t->stride[i];
  return {base, base + (uintptr_t)((last + 1) * (int64_t)elem_size(t->dtype))};
}
bool empty(const ttt_tensor* t) {
  for (int i = 0; i < t->ndim; ++i)
    if (t->shape[i] == 0) return true;
  return false;
}
bool overlaps(const ttt_tensor* a, const ttt_tensor* b) {
  if (!a || !b || empty(a) || empty(b)) return false;
  Extent x = extent(a), y = extent(b);
  return x.lo < y.hi && y.lo < x.hi;
}

bool contiguous(const ttt_tensor* t) {
  int64_t s = 1;
  for (int i = t->ndim - 1; i >= 0; --i) {
    if (t->shape[i] != 1 && t->stride[i] != s) return false;
    s *= t->shape[i];
  }
  return true;
}

ttt_status check_tokens(const ttt_tensor* t, int64_t B, int64_t H, int64_t T, int64_t d,
                        int32_t dtype) {
  if (!t->data && !(B * H * T * d == 0)) return TTT_ERR_NULL;
  if (t->ndim != 4) return TTT_ERR_SHAPE;
  if (t->shape[0] != B || t->shape[1] != H || t->shape[2] != T || t->shape[3] != d)
    return TTT_ERR_SHAPE;
  if (t->dtype != dtype) return TTT_ERR_DTYPE;
  if (B * H * T * d == 0) return TTT_OK;  // no elements: strides are irrelevant
  if (t->stride[3] != 1 && d > 1) return TTT_ERR_LAYOUT;
  const int64_t es = (int64_t)elem_size(dtype);
  for (int i = 0; i < 3; ++i) {
    if (t->stride[i] < 0) return TTT_ERR_LAYOUT;
    if ((t->stride[i] * es) % 16 != 0 && t->shape[i] > 1) return TTT_ERR_LAYOUT;
  }
  if (!aligned16(t->data)) return TTT_ERR_LAYOUT;
  return TTT_OK;
}

ttt::TokView view(const ttt_tensor* t) { return {t->data, t->stride[0], t->stride[1], t->stride[2]}; }

ttt_status lact_check_weight(const ttt_tensor* W, int64_t B, int64_t H, int64_t r,
                                    int64_t c, int64_t* sb) {
  if (!W->data) return TTT_ERR_NULL;
  if (W->dtype != TTT_F32) return TTT_ERR_DTYPE;
  if (W->ndim == 3) {
    if (W->shape[0] != H || W->shape[1] != r || W->shape[2] != c) return TTT_ERR_SHAPE;
    *sb = 0;
  } else if (W->ndim == 4) {
    if (W->shape[0] != B || W->shape[1] != H || W->shape[2] != r || W->shape[3] != c)
      return TTT_ERR_SHAPE;
    *sb = H * r * c;
  } else {
    return TTT_ERR_SHAPE;
  }
  if (!contiguous(W) || !aligned16(W->data)) return TTT_ERR_LAYOUT;
  return TTT_OK;
}

ttt_status lact_check_final(const ttt_tensor* W, int64_t B, int64_t H, int64_t r,
                                   int64_t c) {
  if (!W) return TTT_OK;
  if (!W->data) return TTT_ERR_NULL;
  if (W->dtype != TTT_F32) return TTT_ERR_DTYPE;
  if (W->ndim != 4 || W->shape[0] != B || W->shape[1] != H || W->shape[2] != r ||
      W->shape[3] != c)
    return TTT_ERR_SHAPE;
  if (!contiguous(W) || !aligned16(W->data)) return TTT_ERR_LAYOUT;
  return TTT_OK;
}

// Failure-detection self-test: one thread waits on a barrier that nothing
// arrives at. The bounded wait gives up after its time limit, records the
// timeout in the status word and the kernel returns (no trap, no hang).
__global__ void selftest_wait_kernel(int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ttt::mbar_init(&bar, 1);
    ttt::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) ttt::mbar_wait(&bar, 0, status);
}

// Debug-bounds self-test: one index check that fails by construction (no
// memory is accessed); the debug-bounds build records TTT_ERR_BOUNDS.
__global__ void selftest_bounds_kernel(int* status) {
  if (!TTT_BOUNDS(threadIdx.x > 1024u, status)) return;
}

}  // namespace

extern "C" {

int32_t ttt_version(void) { return 200; }

ttt_status ttt_selftest_bounds(void* stream) {
#ifdef TTT_DEBUG_BOUNDS
  int* p = device_status_ptr();
  if (!p) return TTT_ERR_CUDA;
  selftest_bounds_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
#else
  (void)stream;
  return TTT_ERR_UNSUPPORTED;  // the checks are compiled out of this build
#endif
}

void ttt_test_fail_allocations(int32_t n) { ttt::set_failing_allocs(n); }

ttt_status ttt_selftest_wait_timeout(void* stream) {
  int* p = device_status_ptr();
  if (!p) return TTT_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

const char* ttt_status_string(int32_t s) {
  switch (s) {
    case TTT_OK: return "ok";
    case TTT_ERR_NULL: return "a required pointer is NULL";
    case TTT_ERR_SHAPE: return "tensor shapes are inconsistent or have the wrong rank";
    case TTT_ERR_DTYPE: return "element type not allowed for this tensor";
    case TTT_ERR_LAYOUT: return "stride or 16-byte alignment rule broken";
    case TTT_ERR_UNSUPPORTED: return "no kernel in this library for these sizes/types";
    case TTT_ERR_CUDA: return "a CUDA runtime call failed";
    case TTT_ERR_TIMEOUT: return "a device-side bounded wait gave up";
    case TTT_ERR_ALLOC: return "stream-ordered scratch allocation failed";
    case TTT_ERR_ARG: return "scalar argument out of range";
    case TTT_ERR_SCRATCH: return "scratch need exceeds the fixed pool of lact_swiglu_fwd_noalloc";
    case TTT_ERR_BOUNDS: return "a kernel index check of the debug-bounds build failed";
    default: return "unknown status";
  }
}

ttt_status ttt_get_device_status(void* stream) {
  int* p = device_status_ptr();
  if (!p) return TTT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return TTT_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ERR_CUDA;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return TTT_ERR_CUDA;
  if (v == ttt::DEV_TIMEOUT) return TTT_ERR_TIMEOUT;
  if (v == ttt::DEV_BOUNDS) return TTT_ERR_BOUNDS;
  if (v != ttt::DEV_OK) return TTT_ERR_CUDA;
  return TTT_OK;
}

ttt_status ttt_linear_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                          const ttt_tensor* eta, const ttt_tensor* W0, int32_t chunk,
                          int32_t loss, const ttt_tensor* out, const ttt_tensor* W_final,
                          void* stream) {
  if (!q || !k || !v || !eta || !W0 || !out) return TTT_ERR_NULL;
  if (chunk < 1) return TTT_ERR_ARG;
  if (loss != TTT_LOSS_MSE && loss != TTT_LOSS_NEG_DOT) return TTT_ERR_ARG;
  if (q->ndim != 4 || v->ndim != 4) return TTT_ERR_SHAPE;
  const int64_t B = q->shape[0], H = q->shape[1], T = q->shape[2], dk = q->shape[3];
  const int64_t dv = v->shape[3];
  if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1) return TTT_ERR_SHAPE;
  if (dk > 256 || dv > 256 || T > kMaxT || B * H > kMaxHeads) return TTT_ERR_UNSUPPORTED;
  const int32_t dt = q->dtype;
  if (dt != TTT_F32 && dt != TTT_BF16) return TTT_ERR_DTYPE;
  ttt_status st;
  if ((st = check_tokens(q, B, H, T, dk, dt)) != TTT_OK) return st;
  if ((st = check_tokens(k, B, H, T, dk, dt)) != TTT_OK) return st;
  if ((st = check_tokens(v, B, H, T, dv, dt)) != TTT_OK) return st;
  if ((st = check_tokens(out, B, H, T, dv, dt)) != TTT_OK) return st;
  // eta [B,H,T] fp32, any non-negative strides
  if (eta->ndim != 3 || eta->shape[0] != B || eta->shape[1] != H || eta->shape[2] != T)
    return TTT_ERR_SHAPE;
  if (eta->dtype != TTT_F32) return TTT_ERR_DTYPE;
  if (!eta->data && T > 0) return TTT_ERR_NULL;
  for (int i = 0; i < 3; ++i)
    if (eta->stride[i] < 0 && T > 0) return TTT_ERR_LAYOUT;
  if (!aligned16(eta->data)) return TTT_ERR_LAYOUT;
  // W0 [H,dk,dv] or [B,H,dk,dv] fp32 contiguous
  if (!W0->data) return TTT_ERR_NULL;
  if (W0->dtype != TTT_F32) return TTT_ERR_DTYPE;
  int64_t w0_sb = 0;
  if (W0->ndim == 3) {
    if (W0->shape[0] != H || W0->shape[1] != dk || W0->shape[2] != dv) return TTT_ERR_SHAPE;
  } else if (W0->ndim == 4) {
    if (W0->shape[0] != B || W0->shape[1] != H || W0->shape[2] != dk || W0->shape[3] != dv)
      return TTT_ERR_SHAPE;
    w0_sb = H * dk * dv;
  } else {
    return TTT_ERR_SHAPE;
  }
  if (!contiguous(W0) || !aligned16(W0->data)) return TTT_ERR_LAYOUT;
  if (W_final) {
    if (!W_final->data) return TTT_ERR_NULL;
    if (W_final->dtype != TTT_F32) return TTT_ERR_DTYPE;
    if (W_final->ndim != 4 || W_final->shape[0] != B || W_final->shape[1] != H ||
        W_final->shape[2] != dk || W_final->shape[3] != dv)
      return TTT_ERR_SHAPE;
    if (!contiguous(W_final) || !aligned16(W_final->data)) return TTT_ERR_LAYOUT;
  }
  const ttt_tensor* ins[] = {q, k, v, eta, W0};
  for (const ttt_tensor* in : ins)
    if (overlaps(out, in) || overlaps(W_final, in)) return TTT_ERR_ARG;
  if (overlaps(out, W_final)) return TTT_ERR_ARG;

  ttt::LinearArgs a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.eta = {static_cast<const float*>(eta->data), eta->stride[0], eta->stride[1], eta->stride[2]};
  a.W0 = static_cast<const float*>(W0->data);
  a.w0_sb = w0_sb;
  a.out = {out->data, out->stride[0], out->stride[1], out->stride[2]};
  a.W_final = W_final ? static_cast<float*>(W_final->data) : nullptr;
  a.B = (int)B;
  a.H = (int)H;
  a.T = (int)T;
  a.dk = (int)dk;
  a.dv = (int)dv;
  a.chunk = chunk;
  a.loss = loss;
  a.status = device_status_ptr();
  if (!a.status) return TTT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaError_t e;
  if (dt == TTT_F32 || T == 0) {  // T == 0 only copies W0 to W_final
    e = ttt::launch_ttt_linear_f32(a, s);
  } else {
    bool supported = false;
    e = ttt::launch_ttt_linear_bf16(a, s, &supported);
    if (!supported) return TTT_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

}  // extern "C"

namespace ttt {

ttt_status lact_build_args(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                           const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                           const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                           int32_t causal, const ttt_tensor* out, const ttt_tensor* W1_final,
                           const ttt_tensor* W2_final, const ttt_tensor* W3_final, LactArgs* ap) {
  if (!q || !k || !v || !eta || !W1 || !W2 || !W3 || !out) return TTT_ERR_NULL;
  if (chunk < 1) return TTT_ERR_ARG;
  if (update_rule != LACT_UPDATE_GD && update_rule != LACT_UPDATE_MUON) return TTT_ERR_ARG;
  if (causal != 0 && causal != 1) return TTT_ERR_ARG;
  if (q->ndim != 4 || v->ndim != 4 || W1->ndim < 3) return TTT_ERR_SHAPE;
  const int64_t B = q->shape[0], H = q->shape[1], T = q->shape[2], dk = q->shape[3];
  const int64_t dv = v->shape[3];
  const int64_t dh = W1->shape[W1->ndim - 2];
  if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1 || dh < 1) return TTT_ERR_SHAPE;
  if (dk > 256 || dv > 256 || dh > 4096 || T > kMaxT || B * H > kMaxHeads)
    return TTT_ERR_UNSUPPORTED;
  const int32_t dt = q->dtype;
  if (dt != TTT_F32 && dt != TTT_BF16) return TTT_ERR_DTYPE;
  ttt_status st;
  if ((st = check_tokens(q, B, H, T, dk, dt)) != TTT_OK) return st;
  if ((st = check_tokens(k, B, H, T, dk, dt)) != TTT_OK) return st;
  if ((st = check_tokens(v, B, H, T, dv, dt)) != TTT_OK) return st;
  if ((st = check_tokens(out, B, H, T, dv, dt)) != TTT_OK) return st;
  if (eta->ndim != 3 || eta->shape[0] != B || eta->shape[1] != H || eta->shape[2] != T)
    return TTT_ERR_SHAPE;
  if (eta->dtype != TTT_F32) return TTT_ERR_DTYPE;
  if (!eta->data && T > 0) return TTT_ERR_NULL;
  for (int i = 0; i < 3; ++i)
    if (eta->stride[i] < 0) return TTT_ERR_LAYOUT;
  if (!aligned16(eta->data)) return TTT_ERR_LAYOUT;
  int64_t sb1, sb2, sb3;
  if ((st = lact_check_weight(W1, B, H, dh, dk, &sb1)) != TTT_OK) return st;
  if ((st = lact_check_weight(W2, B, H, dv, dh, &sb2)) != TTT_OK) return st;
  if ((st = lact_check_weight(W3, B, H, dh, dk, &sb3)) != TTT_OK) return st;
  if ((st = lact_check_final(W1_final, B, H, dh, dk)) != TTT_OK) return st;
  if ((st = lact_check_final(W2_final, B, H, dv, dh)) != TTT_OK) return st;
  if ((st = lact_check_final(W3_final, B, H, dh, dk)) != TTT_OK) return st;
  const ttt_tensor* ins[] = {q, k, v, eta, W1, W2, W3};
  const ttt_tensor* outs[] = {out, W1_final, W2_final, W3_final};
  for (const ttt_tensor* o : outs) {
    for (const ttt_tensor* in : ins)
      if (overlaps(o, in)) return TTT_ERR_ARG;
    for (const ttt_tensor* o2 : outs)
      if (o != o2 && overlaps(o, o2)) return TTT_ERR_ARG;
  }

  LactArgs& a = *ap;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.eta = {static_cast<const float*>(eta->data), eta->stride[0], eta->stride[1], eta->stride[2]};
  a.W1 = static_cast<const float*>(W1->data);
  a.W2 = static_cast<const float*>(W2->data);
  a.W3 = static_cast<const float*>(W3->data);
  a.w_sb[0] = sb1;
  a.w_sb[1] = sb2;
  a.w_sb[2] = sb3;
  a.out = {out->data, out->stride[0], out->stride[1], out->stride[2]};
  a.W1_final = W1_final ? static_cast<float*>(W1_final->data) : nullptr;
  a.W2_final = W2_final ? static_cast<float*>(W2_final->data) : nullptr;
  a.W3_final = W3_final ? static_cast<float*>(W3_final->data) : nullptr;
  a.B = (int)B;
  a.H = (int)H;
  a.T = (int)T;
  a.dk = (int)dk;
  a.dv = (int)dv;
  a.dh = (int)dh;
  a.chunk = chunk;
  a.update_rule = update_rule;
  a.causal = causal;
  a.dtype = dt;
  a.status = nullptr;
  a.momentum = 0;
  a.beta = 0.f;
  a.reduce = nullptr;
  a.reduce_user = nullptr;
  for (int m = 0; m < 3; ++m) {
    a.M0[m] = nullptr;
    a.m0_sb[m] = 0;
    a.M_final[m] = nullptr;
  }
  return TTT_OK;
}

ttt_status lact_attach_status(LactArgs* a) {
  a->status = device_status_ptr();
  return a->status ? TTT_OK : TTT_ERR_CUDA;
}

}  // namespace ttt

extern "C" {

ttt_status lact_swiglu_fwd_ex(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                              const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                              const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                              int32_t causal, const ttt_tensor* out,
                              const ttt_tensor* W1_final, const ttt_tensor* W2_final,
                              const ttt_tensor* W3_final, void* stream) {
  ttt::LactArgs a;
  ttt_status st = ttt::lact_build_args(q, k, v, eta, W1, W2, W3, chunk, update_rule, causal, out,
                                       W1_final, W2_final, W3_final, &a);
  if (st != TTT_OK) return st;
  if ((st = ttt::lact_attach_status(&a)) != TTT_OK) return st;
  return ttt::lact_forward(a, static_cast<cudaStream_t>(stream));
}

ttt_status lact_swiglu_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                           const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                           const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                           int32_t causal, const ttt_tensor* out, void* stream) {
  return lact_swiglu_fwd_ex(q, k, v, eta, W1, W2, W3, chunk, update_rule, causal, out, nullptr,
                            nullptr, nullptr, stream);
}

}  // extern "C"

extern "C" {

ttt_status lact_swiglu_fwd_momentum(const ttt_tensor* q, const ttt_tensor* k,
                                    const ttt_tensor* v, const ttt_tensor* eta,
                                    const ttt_tensor* W1, const ttt_tensor* W2,
                                    const ttt_tensor* W3, int32_t chunk, float beta,
                                    int32_t causal, const ttt_tensor* M1_0,
                                    const ttt_tensor* M2_0, const ttt_tensor* M3_0,
                                    const ttt_tensor* out, const ttt_tensor* W1_final,
                                    const ttt_tensor* W2_final, const ttt_tensor* W3_final,
                                    const ttt_tensor* M1_final, const ttt_tensor* M2_final,
                                    const ttt_tensor* M3_final, void* stream) {
  ttt::LactArgs a;
  ttt_status st = ttt::lact_build_args(q, k, v, eta, W1, W2, W3, chunk, LACT_UPDATE_GD, causal,
                                       out, W1_final, W2_final, W3_final, &a);
  if (st != TTT_OK) return st;
  if (!(beta == beta) || beta < -1e30f || beta > 1e30f) return TTT_ERR_ARG;  // finite
  const int64_t B = a.B, H = a.H, dk = a.dk, dv = a.dv, dh = a.dh;
  const ttt_tensor* M0[3] = {M1_0, M2_0, M3_0};
  const ttt_tensor* Mf[3] = {M1_final, M2_final, M3_final};
  const int64_t rows[3] = {dh, dv, dh}, cols[3] = {dk, dh, dk};
  for (int m = 0; m < 3; ++m) {
    if (M0[m]) {
      int64_t sb = 0;
      if ((st = lact_check_weight(M0[m], B, H, rows[m], cols[m], &sb)) != TTT_OK) return st;
      a.M0[m] = static_cast<const float*>(M0[m]->data);
      a.m0_sb[m] = sb;
    }
    if ((st = lact_check_final(Mf[m], B, H, rows[m], cols[m])) != TTT_OK) return st;
    a.M_final[m] = Mf[m] ? static_cast<float*>(Mf[m]->data) : nullptr;
  }
  // outputs overlap no input and no other output
  const ttt_tensor* ins[] = {q, k, v, eta, W1, W2, W3, M1_0, M2_0, M3_0};
  const ttt_tensor* outs[] = {out, W1_final, W2_final, W3_final, M1_final, M2_final, M3_final};
  for (const ttt_tensor* o : outs) {
    for (const ttt_tensor* in : ins)
      if (overlaps(o, in)) return TTT_ERR_ARG;
    for (const ttt_tensor* o2 : outs)
      if (o != o2 && overlaps(o, o2)) return TTT_ERR_ARG;
  }
  a.momentum = 1;
  a.beta = beta;
  if ((st = ttt::lact_attach_status(&a)) != TTT_OK) return st;
  return ttt::lact_forward(a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

extern "C" {

ttt_status ttt_linear_bwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                          const ttt_tensor* eta, const ttt_tensor* W0, int32_t chunk,
                          int32_t loss, const ttt_tensor* dy, const ttt_tensor* dW_final,
                          const ttt_tensor* dq, const ttt_tensor* dk, const ttt_tensor* dv,
                          const ttt_tensor* deta, const ttt_tensor* dW0, void* stream) {
  if (!q || !k || !v || !eta || !W0 || !dy || !dq || !dk || !dv || !deta || !dW0)
    return TTT_ERR_NULL;
  if (chunk < 1) return TTT_ERR_ARG;
  if (loss != TTT_LOSS_MSE && loss != TTT_LOSS_NEG_DOT) return TTT_ERR_ARG;
  if (q->ndim != 4 || v->ndim != 4) return TTT_ERR_SHAPE;
  const int64_t B = q->shape[0], H = q->shape[1], T = q->shape[2], dK = q->shape[3];
  const int64_t dV = v->shape[3];
  if (B < 1 || H < 1 || T < 0 || dK < 1 || dV < 1) return TTT_ERR_SHAPE;
  if (T > kMaxT || B * H > kMaxHeads || !ttt::ttt_linear_bwd_supported((int)dK, (int)dV))
    return TTT_ERR_UNSUPPORTED;
  const int32_t dt = q->dtype;
  if (dt != TTT_F32 && dt != TTT_BF16) return TTT_ERR_DTYPE;
  ttt_status st;
  if ((st = check_tokens(q, B, H, T, dK, dt)) != TTT_OK) return st;
  if ((st = check_tokens(k, B, H, T, dK, dt)) != TTT_OK) return st;
  if ((st = check_tokens(v, B, H, T, dV, dt)) != TTT_OK) return st;
  if ((st = check_tokens(dy, B, H, T, dV, dt)) != TTT_OK) return st;
  if ((st = check_tokens(dq, B, H, T, dK, dt)) != TTT_OK) return st;
  if ((st = check_tokens(dk, B, H, T, dK, dt)) != TTT_OK) return st;
  if ((st = check_tokens(dv, B, H, T, dV, dt)) != TTT_OK) return st;
  auto check_eta = [&](const ttt_tensor* e, bool contig) -> ttt_status {
    if (e->ndim != 3 || e->shape[0] != B || e->shape[1] != H || e->shape[2] != T)
      return TTT_ERR_SHAPE;
    if (e->dtype != TTT_F32) return TTT_ERR_DTYPE;
    if (!e->data && T > 0) return TTT_ERR_NULL;
    for (int i = 0; i < 3; ++i)
      if (e->stride[i] < 0 && T > 0) return TTT_ERR_LAYOUT;
    if (contig && T > 0 && !contiguous(e)) return TTT_ERR_LAYOUT;
    if (!aligned16(e->data)) return TTT_ERR_LAYOUT;
    return TTT_OK;
  };
  if ((st = check_eta(eta, false)) != TTT_OK) return st;
  if ((st = check_eta(deta, true)) != TTT_OK) return st;
  // W0 and dW0: [H,dk,dv] (shared over the batch) or [B,H,dk,dv], fp32 contiguous
  auto check_w = [&](const ttt_tensor* w, int64_t* sb) -> ttt_status {
    if (!w->data) return TTT_ERR_NULL;
    if (w->dtype != TTT_F32) return TTT_ERR_DTYPE;
    if (w->ndim == 3) {
      if (w->shape[0] != H || w->shape[1] != dK || w->shape[2] != dV) return TTT_ERR_SHAPE;
      *sb = 0;
    } else if (w->ndim == 4) {
      if (w->shape[0] != B || w->shape[1] != H || w->shape[2] != dK || w->shape[3] != dV)
        return TTT_ERR_SHAPE;
      *sb = H * dK * dV;
    } else {
      return TTT_ERR_SHAPE;
    }
    if (!contiguous(w) || !aligned16(w->data)) return TTT_ERR_LAYOUT;
    return TTT_OK;
  };
  int64_t w0_sb = 0, dw0_sb = 0;
  if ((st = check_w(W0, &w0_sb)) != TTT_OK) return st;
  if ((st = check_w(dW0, &dw0_sb)) != TTT_OK) return st;
  if (W0->ndim != dW0->ndim) return TTT_ERR_SHAPE;
  if (dW_final) {
    if (!dW_final->data) return TTT_ERR_NULL;
    if (dW_final->dtype != TTT_F32) return TTT_ERR_DTYPE;
    if (dW_final->ndim != 4 || dW_final->shape[0] != B || dW_final->shape[1] != H ||
        dW_final->shape[2] != dK || dW_final->shape[3] != dV)
      return TTT_ERR_SHAPE;
    if (!contiguous(dW_final) || !aligned16(dW_final->data)) return TTT_ERR_LAYOUT;
  }
  const ttt_tensor* ins[] = {q, k, v, eta, W0, dy, dW_final};
  const ttt_tensor* outs[] = {dq, dk, dv, deta, dW0};
  for (const ttt_tensor* o : outs) {
    for (const ttt_tensor* in : ins)
      if (overlaps(o, in)) return TTT_ERR_ARG;
    for (const ttt_tensor* o2 : outs)
      if (o != o2 && overlaps(o, o2)) return TTT_ERR_ARG;
  }

  ttt::LinearBwdArgs a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.dy = view(dy);
  a.eta = {static_cast<const float*>(eta->data), eta->stride[0], eta->stride[1], eta->stride[2]};
  a.W0 = static_cast<const float*>(W0->data);
  a.w0_sb = w0_sb;
  a.dWf = dW_final ? static_cast<const float*>(dW_final->data) : nullptr;
  a.gq = {dq->data, dq->stride[0], dq->stride[1], dq->stride[2]};
  a.gk = {dk->data, dk->stride[0], dk->stride[1], dk->stride[2]};
  a.gv = {dv->data, dv->stride[0], dv->stride[1], dv->stride[2]};
  a.deta = static_cast<float*>(deta->data);
  a.dW = nullptr;
  a.ckpt = nullptr;
  a.B = (int)B;
  a.H = (int)H;
  a.T = (int)T;
  a.dk = (int)dK;
  a.dv = (int)dV;
  a.chunk = chunk;
  a.loss = loss;
  a.nchunks = (int)((T + chunk - 1) / chunk);
  a.status = device_status_ptr();
  if (!a.status) return TTT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool shared = W0->ndim == 3;
  const size_t bytes = ttt::ttt_linear_bwd_workspace(a, shared);
  void* ws = nullptr;
  if (bytes && ttt::scratch_alloc(&ws, bytes, s) != cudaSuccess) return TTT_ERR_ALLOC;
  cudaError_t e = ttt::launch_ttt_linear_bwd(a, dt == TTT_BF16, shared,
                                             static_cast<float*>(dW0->data), ws, s);
  if (ws && cudaFreeAsync(ws, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

}  // extern "C"

namespace {

// Parameter tensor of per-head shape `inner` (1 or 2 dims): [H, inner...] shared
// over the batch, or [B, H, inner...]; fp32 contiguous. *per_seq = 1 for the latter.
ttt_status check_param(const ttt_tensor* t, int64_t B, int64_t H, int nin, const int64_t* inner,
                       int64_t* per_seq) {
  if (!t->data) return TTT_ERR_NULL;
  if (t->dtype != TTT_F32) return TTT_ERR_DTYPE;
  int off;
  if (t->ndim == nin + 1) {
    if (t->shape[0] != H) return TTT_ERR_SHAPE;
    off = 1;
    *per_seq = 0;
  } else if (t->ndim == nin + 2) {
    if (t->shape[0] != B || t->shape[1] != H) return TTT_ERR_SHAPE;
    off = 2;
    *per_seq = 1;
  } else {
    return TTT_ERR_SHAPE;
  }
  for (int i = 0; i < nin; ++i)
    if (t->shape[off + i] != inner[i]) return TTT_ERR_SHAPE;
  if (!contiguous(t) || !aligned16(t->data)) return TTT_ERR_LAYOUT;
  return TTT_OK;
}

ttt_status check_final_param(const ttt_tensor* t, int64_t B, int64_t H, int nin,
                             const int64_t* inner) {
  if (!t) return TTT_OK;
  int64_t per = 0;
  ttt_status st = check_param(t, B, H, nin, inner, &per);
  if (st != TTT_OK) return st;
  return per ? TTT_OK : TTT_ERR_SHAPE;
}

}  // namespace

extern "C" {

ttt_status ttt_mlp_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                       const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* b1,
                       const ttt_tensor* W2, const ttt_tensor* b2, int32_t chunk,
                       const ttt_tensor* out, const ttt_tensor* W1_final,
                       const ttt_tensor* b1_final, const ttt_tensor* W2_final,
                       const ttt_tensor* b2_final, void* stream) {
  if (!q || !k || !v || !eta || !W1 || !b1 || !W2 || !b2 || !out) return TTT_ERR_NULL;
  if (chunk < 1) return TTT_ERR_ARG;
  if (q->ndim != 4 || v->ndim != 4 || W1->ndim < 3) return TTT_ERR_SHAPE;
  const int64_t B = q->shape[0], H = q->shape[1], T = q->shape[2], dK = q->shape[3];
  const int64_t dV = v->shape[3], dH = W1->shape[W1->ndim - 2];
  if (B < 1 || H < 1 || T < 0 || dK < 1 || dV < 1 || dH < 1) return TTT_ERR_SHAPE;
  if (T > kMaxT || B * H > kMaxHeads || !ttt::ttt_mlp_supported((int)dK, (int)dV, (int)dH))
    return TTT_ERR_UNSUPPORTED;
  const int32_t dt = q->dtype;
  if (dt != TTT_F32 && dt != TTT_BF16) return TTT_ERR_DTYPE;
  ttt_status st;
  if ((st = check_tokens(q, B, H, T, dK, dt)) != TTT_OK) return st;
  if ((st = check_tokens(k, B, H, T, dK, dt)) != TTT_OK) return st;
  if ((st = check_tokens(v, B, H, T, dV, dt)) != TTT_OK) return st;
  if ((st = check_tokens(out, B, H, T, dV, dt)) != TTT_OK) return st;
  if (eta->ndim != 3 || eta->shape[0] != B || eta->shape[1] != H || eta->shape[2] != T)
    return TTT_ERR_SHAPE;
  if (eta->dtype != TTT_F32) return TTT_ERR_DTYPE;
  if (!eta->data && T > 0) return TTT_ERR_NULL;
  for (int i = 0; i < 3; ++i)
    if (eta->stride[i] < 0) return TTT_ERR_LAYOUT;
  if (!aligned16(eta->data)) return TTT_ERR_LAYOUT;
  const int64_t sW1[2] = {dH, dK}, sb1[1] = {dH}, sW2[2] = {dV, dH}, sb2[1] = {dV};
  const ttt_tensor* P[4] = {W1, b1, W2, b2};
  const ttt_tensor* F[4] = {W1_final, b1_final, W2_final, b2_final};
  const int64_t* inner[4] = {sW1, sb1, sW2, sb2};
  const int nin[4] = {2, 1, 2, 1};
  int64_t per[4];
  for (int m = 0; m < 4; ++m) {
    if ((st = check_param(P[m], B, H, nin[m], inner[m], &per[m])) != TTT_OK) return st;
    if ((st = check_final_param(F[m], B, H, nin[m], inner[m])) != TTT_OK) return st;
  }
  const ttt_tensor* ins[] = {q, k, v, eta, W1, b1, W2, b2};
  const ttt_tensor* outs[] = {out, W1_final, b1_final, W2_final, b2_final};
  for (const ttt_tensor* o : outs) {
    for (const ttt_tensor* in : ins)
      if (overlaps(o, in)) return TTT_ERR_ARG;
    for (const ttt_tensor* o2 : outs)
      if (o != o2 && overlaps(o, o2)) return TTT_ERR_ARG;
  }
  ttt::MlpArgs a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.eta = {static_cast<const float*>(eta->data), eta->stride[0], eta->stride[1], eta->stride[2]};
  a.W1 = static_cast<const float*>(W1->data);
  a.b1 = static_cast<const float*>(b1->data);
  a.W2 = static_cast<const float*>(W2->data);
  a.b2 = static_cast<const float*>(b2->data);
  for (int m = 0; m < 4; ++m) a.p_sb[m] = per[m];
  a.out = {out->data, out->stride[0], out->stride[1], out->stride[2]};
  float* fin[4];
  for (int m = 0; m < 4; ++m) fin[m] = F[m] ? static_cast<float*>(F[m]->data) : nullptr;
  a.W1_final = fin[0];
  a.b1_final = fin[1];
  a.W2_final = fin[2];
  a.b2_final = fin[3];
  a.B = (int)B;
  a.H = (int)H;
  a.T = (int)T;
  a.dk = (int)dK;
  a.dv = (int)dV;
  a.dh = (int)dH;
  a.chunk = chunk;
  a.status = device_status_ptr();
  if (!a.status) return TTT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = ttt::ttt_mlp_workspace(a);
  void* ws = nullptr;
  if (ttt::scratch_alloc(&ws, bytes, s) != cudaSuccess) return TTT_ERR_ALLOC;
  a.ws = static_cast<float*>(ws);
  cudaError_t e = ttt::launch_ttt_mlp(a, dt == TTT_BF16, s);
  if (cudaFreeAsync(ws, s) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

}  // extern "C"

extern "C" {

ttt_status window_attention_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                                int32_t window, int32_t accumulate, const ttt_tensor* out,
                                void* stream) {
  if (!q || !k || !v || !out) return TTT_ERR_NULL;
  if (window < 1 || (accumulate != 0 && accumulate != 1)) return TTT_ERR_ARG;
  if (q->ndim != 4 || v->ndim != 4) return TTT_ERR_SHAPE;
  const int64_t B = q->shape[0], H = q->shape[1], T = q->shape[2], d = q->shape[3];
  const int64_t dV = v->shape[3];
  if (B < 1 || H < 1 || T < 0 || d < 1 || dV < 1) return TTT_ERR_SHAPE;
  const int32_t dt = q->dtype;
  if (dt != TTT_F32 && dt != TTT_BF16) return TTT_ERR_DTYPE;
  ttt_status st;
  if ((st = check_tokens(q, B, H, T, d, dt)) != TTT_OK) return st;
  if ((st = check_tokens(k, B, H, T, d, dt)) != TTT_OK) return st;
  if ((st = check_tokens(v, B, H, T, dV, dt)) != TTT_OK) return st;
  if ((st = check_tokens(out, B, H, T, dV, dt)) != TTT_OK) return st;
  if (T > kMaxT || B * H > kMaxHeads || !ttt::window_attn_supported((int)d, (int)dV, dt))
    return TTT_ERR_UNSUPPORTED;
  if (overlaps(out, q) || overlaps(out, k) || overlaps(out, v)) return TTT_ERR_ARG;
  cudaError_t e = ttt::launch_window_attn(view(q), view(k), view(v),
                                          {out->data, out->stride[0], out->stride[1], out->stride[2]},
                                          (int)B, (int)H, (int)T, (int)d, window, accumulate,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

ttt_status lact_swiglu_window_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                                  const ttt_tensor* eta, const ttt_tensor* W1,
                                  const ttt_tensor* W2, const ttt_tensor* W3, int32_t chunk,
                                  int32_t update_rule, int32_t window, const ttt_tensor* out,
                                  void* stream) {
  if (!q || !v || !out) return TTT_ERR_NULL;
  if (window < 1) return TTT_ERR_ARG;
  if (q->ndim != 4 || v->ndim != 4) return TTT_ERR_SHAPE;
  if (!ttt::window_attn_supported((int)q->shape[3], (int)v->shape[3], q->dtype))
    return TTT_ERR_UNSUPPORTED;
  ttt_status st = lact_swiglu_fwd(q, k, v, eta, W1, W2, W3, chunk, update_rule, 1, out, stream);
  if (st != TTT_OK) return st;
  return window_attention_fwd(q, k, v, window, 1, out, stream);
}

}  // extern "C"

extern "C" {

ttt_status lact_swiglu_fwd_cp(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                              const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                              const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                              int32_t causal, const ttt_tensor* out,
                              const ttt_tensor* W1_final, const ttt_tensor* W2_final,
                              const ttt_tensor* W3_final, lact_grad_reduce_fn reduce,
                              void* reduce_user, void* stream) {
  ttt::LactArgs a;
  ttt_status st = ttt::lact_build_args(q, k, v, eta, W1, W2, W3, chunk, update_rule, causal, out,
                                       W1_final, W2_final, W3_final, &a);
  if (st != TTT_OK) return st;
  a.reduce = reduce;
  a.reduce_user = reduce_user;
  if ((st = ttt::lact_attach_status(&a)) != TTT_OK) return st;
  return ttt::lact_forward(a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

extern "C" {

ttt_status lact_swiglu_bwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                           const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                           const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                           int32_t causal, const ttt_tensor* dy, const ttt_tensor* dW1_final,
                           const ttt_tensor* dW2_final, const ttt_tensor* dW3_final,
                           const ttt_tensor* dq, const ttt_tensor* dk, const ttt_tensor* dv,
                           const ttt_tensor* deta, const ttt_tensor* dW1, const ttt_tensor* dW2,
                           const ttt_tensor* dW3, void* stream) {
  if (!dy || !dq || !dk || !dv || !deta || !dW1 || !dW2 || !dW3) return TTT_ERR_NULL;
  ttt::LactArgs a;
  // the forward's arguments, with dy in the place of the output (same shape)
  ttt_status st = ttt::lact_build_args(q, k, v, eta, W1, W2, W3, chunk, update_rule, causal, dy,
                                       nullptr, nullptr, nullptr, &a);
  if (st != TTT_OK) return st;
  if (!ttt::lact_bwd_supported(a)) return TTT_ERR_UNSUPPORTED;
  const int64_t B = a.B, H = a.H, T = a.T, dK = a.dk, dV = a.dv, dH = a.dh;
  if ((st = check_tokens(dq, B, H, T, dK, a.dtype)) != TTT_OK) return st;
  if ((st = check_tokens(dk, B, H, T, dK, a.dtype)) != TTT_OK) return st;
  if ((st = check_tokens(dv, B, H, T, dV, a.dtype)) != TTT_OK) return st;
  if (deta->ndim != 3 || deta->shape[0] != B || deta->shape[1] != H || deta->shape[2] != T)
    return TTT_ERR_SHAPE;
  if (deta->dtype != TTT_F32) return TTT_ERR_DTYPE;
  if (!deta->data && T > 0) return TTT_ERR_NULL;
  if (T > 0 && (!contiguous(deta) || !aligned16(deta->data))) return TTT_ERR_LAYOUT;
  const ttt_tensor* Wt[3] = {W1, W2, W3};
  const ttt_tensor* dWt[3] = {dW1, dW2, dW3};
  const ttt_tensor* dWf[3] = {dW1_final, dW2_final, dW3_final};
  const int64_t rows[3] = {dH, dV, dH}, cols[3] = {dK, dH, dK};
  for (int m = 0; m < 3; ++m) {
    int64_t sb = 0;
    if ((st = lact_check_weight(dWt[m], B, H, rows[m], cols[m], &sb)) != TTT_OK) return st;
    if (dWt[m]->ndim != Wt[m]->ndim) return TTT_ERR_SHAPE;
    if ((st = lact_check_final(dWf[m], B, H, rows[m], cols[m])) != TTT_OK) return st;
  }
  const ttt_tensor* ins[] = {q, k, v, eta, W1, W2, W3, dy, dW1_final, dW2_final, dW3_final};
  const ttt_tensor* outs[] = {dq, dk, dv, deta, dW1, dW2, dW3};
  for (const ttt_tensor* o : outs) {
    for (const ttt_tensor* in : ins)
      if (overlaps(o, in)) return TTT_ERR_ARG;
    for (const ttt_tensor* o2 : outs)
      if (o != o2 && overlaps(o, o2)) return TTT_ERR_ARG;
  }
  ttt::LactBwdArgs g;
  g.dy = view(dy);
  g.dW1_final = dW1_final ? static_cast<const float*>(dW1_final->data) : nullptr;
  g.dW2_final = dW2_final ? static_cast<const float*>(dW2_final->data) : nullptr;
  g.dW3_final = dW3_final ? static_cast<const float*>(dW3_final->data) : nullptr;
  g.dq = {dq->data, dq->stride[0], dq->stride[1], dq->stride[2]};
  g.dk = {dk->data, dk->stride[0], dk->stride[1], dk->stride[2]};
  g.dv = {dv->data, dv->stride[0], dv->stride[1], dv->stride[2]};
  g.deta = static_cast<float*>(deta->data);
  g.dW1 = static_cast<float*>(dW1->data);
  g.dW2 = static_cast<float*>(dW2->data);
  g.dW3 = static_cast<float*>(dW3->data);
  if ((st = ttt::lact_attach_status(&a)) != TTT_OK) return st;
  return ttt::lact_backward(a, g, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
