// LaCT SwiGLU forward on a fixed, library-owned device scratch pool: the one
// entry point of this library that allocates nothing.
//
// Why: lact_swiglu_fwd takes its scratch (fast-weight masters, bf16 operand
// copies, per-chunk activations and gradients) from the device's
// stream-ordered memory pool. Some callers cannot allow that: serving engines
// and training frameworks that reserve (nearly) all device memory up front in
// their own allocator, where an allocation outside it fails or fragments
// memory, and latency-critical loops that must not contain allocation calls.
// This entry point uses instead a file-scope __device__ array of
// kLactPoolBytes, which every device that loads the library holds until the
// process exits.
#include <mutex>

#include "lact.cuh"

namespace {

constexpr size_t kLactPoolBytes = size_t(32) << 20;  // 32 MiB

// The scratch pool. In host code this name is only a handle: its device
// address comes from cudaGetSymbolAddress (per device) below.
static __device__ __align__(256) unsigned char g_lact_pool[kLactPoolBytes];

constexpr int kMaxDevices = 64;
void* g_pool_ptr[kMaxDevices] = {};
std::mutex g_pool_mu;

// Device address of the pool on the current device, looked up once per device
// (on the first call made with that device current).
void* pool_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_pool_mu);
  if (!g_pool_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lact_pool) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_pool_ptr[dev] = p;
  }
  return g_pool_ptr[dev];
}

}  // namespace

extern "C" ttt_status lact_swiglu_fwd_noalloc(
    const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v, const ttt_tensor* eta,
    const ttt_tensor* W1, const ttt_tensor* W2, const ttt_tensor* W3, int32_t chunk,
    int32_t update_rule, int32_t causal, const ttt_tensor* out, const ttt_tensor* W1_final,
    const ttt_tensor* W2_final, const ttt_tensor* W3_final, void* stream) {
  ttt::LactArgs a;
  ttt_status st = ttt::lact_build_args(q, k, v, eta, W1, W2, W3, chunk, update_rule, causal, out,
                                       W1_final, W2_final, W3_final, &a);
  if (st != TTT_OK) return st;
  const size_t need = ttt::lact_scratch_bytes(a);
  if (need == 0) return TTT_ERR_UNSUPPORTED;
  if (need > kLactPoolBytes) return TTT_ERR_SCRATCH;
  if ((st = ttt::lact_attach_status(&a)) != TTT_OK) return st;
  void* pool = pool_ptr();
  if (!pool) return TTT_ERR_CUDA;
  // Every buffer the scan reads is written earlier in the same call (the
  // gradient accumulators are zeroed by its first kernel), so whatever an
  // earlier call left in the pool does not matter.
  return ttt::lact_run(a, static_cast<cudaStream_t>(stream), pool, kLactPoolBytes);
}
