// Shared device/host helpers of libttt_b200 (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/ttt.h"

namespace ttt {

// Error codes a kernel can record in the device status word.
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BAD_ARGS = 2, DEV_BOUNDS = 3 };

// A wait on one barrier gives up after this many nanoseconds of %globaltimer
// (legitimate waits in these kernels last microseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, DEV_OK, code);
}

// Index checks of the debug-bounds build (compiled with -DTTT_DEBUG_BOUNDS):
// TTT_BOUNDS(cond, status) is `cond`, and a false `cond` also records
// DEV_BOUNDS in the status word; the caller skips the access (no trap). In the
// normal build it is the constant `true`, so the checks compile away.
__device__ __forceinline__ bool bounds_check(bool ok, int* status) {
  if (!ok) record_error(status, DEV_BOUNDS);
  return ok;
}
#ifdef TTT_DEBUG_BOUNDS
#define TTT_BOUNDS(cond, status) (::ttt::bounds_check(static_cast<bool>(cond), (status)))
#else
#define TTT_BOUNDS(cond, status) true
#endif

// Strided view of a [B,H,T,d] token tensor (element strides, last stride 1).
struct TokView {
  const void* p;
  int64_t sb, sh, st;
};
struct TokViewMut {
  void* p;
  int64_t sb, sh, st;
};
struct EtaView {
  const float* p;
  int64_t sb, sh, st;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// ---- mbarrier / async-proxy primitives (inline PTX) -------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and records DEV_TIMEOUT) if the phase has not
// completed within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 0 && global_ns() - t0 > kWaitLimitNs) break;
  }
  record_error(status, DEV_TIMEOUT);
  return false;
}

// Programmatic dependent launch: a kernel launched with launch_pdl() may
// start while its predecessor on the stream finishes; it runs its prologue
// (barrier init, TMEM allocation) and then waits here until the predecessor
// has completed and its memory is visible. The trigger lets the next kernel
// of the stream be scheduled early in the same way.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace ttt

// Host-side launchers implemented in the kernel translation units.
namespace ttt {

struct LinearArgs {
  TokView q, k, v;
  EtaView eta;
  const float* W0;
  int64_t w0_sb;   // 0 when W0 is shared over the batch
  TokViewMut out;
  float* W_final;  // may be null
  int B, H, T, dk, dv, chunk, loss;
  int* status;
};

cudaError_t launch_ttt_linear_f32(const LinearArgs& a, cudaStream_t s);
cudaError_t launch_ttt_linear_cc_bf16(const LinearArgs& a, cudaStream_t s);
cudaError_t launch_ttt_linear_bf16(const LinearArgs& a, cudaStream_t s, bool* supported);
bool ttt_linear_wy_supported(const LinearArgs& a);
cudaError_t launch_ttt_linear_wy(const LinearArgs& a, cudaStream_t s);
bool la_tc_supported(const LinearArgs& a);
cudaError_t launch_la_tc(const LinearArgs& a, cudaStream_t s);

// The library's stream-ordered scratch pool on the current device (null if
// it cannot be created; callers then use the device's default pool).
cudaMemPool_t scratch_pool();
// Stream-ordered scratch from that pool (the failure test hook applies).
cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t s);
void set_failing_allocs(int n);

bool window_attn_supported(int d, int dv, int dtype);
cudaError_t launch_window_attn(const TokView& q, const TokView& k, const TokView& v,
                               const TokViewMut& out, int B, int H, int T, int d, int window,
                               int accumulate, cudaStream_t s);

// Arguments of the TTT-MLP forward (ttt_mlp_fwd).
struct MlpArgs {
  TokView q, k, v;
  EtaView eta;
  const float *W1, *b1, *W2, *b2;   // [H or B*H] x ([dh][dk], [dh], [dv][dh], [dv])
  int64_t p_sb[4];                  // non-zero: one copy per (batch, head)
  TokViewMut out;
  float *W1_final, *b1_final, *W2_final, *b2_final;  // [B*H] x ..., each may be null
  float* ws;                        // ttt_mlp_workspace() bytes
  int B, H, T, dk, dv, dh, chunk;
  int* status;
};
bool ttt_mlp_supported(int dk, int dv, int dh);
size_t ttt_mlp_workspace(const MlpArgs& a);
cudaError_t launch_ttt_mlp(const MlpArgs& a, bool bf16, cudaStream_t s);

// Arguments of the TTT-Linear / inner-product backward (ttt_linear_bwd).
struct LinearBwdArgs {
  TokView q, k, v, dy;
  EtaView eta;
  const float* W0;
  int64_t w0_sb;        // 0 when W0 is shared over the batch
  const float* dWf;     // [B,H,dk,dv] or null
  TokViewMut gq, gk, gv;     // dL/dq, dL/dk, dL/dv (same element type as q)
  float* deta;          // [B,H,T] contiguous
  float* dW;            // [B*H][dk][dv]: dL/dW0 per (batch, head)
  float* ckpt;          // [B*H][nchunks][dk][dv] chunk-start weights (MSE)
  int B, H, T, dk, dv, chunk, loss, nchunks;
  int* status;
};

bool ttt_linear_bwd_supported(int dk, int dv);
size_t ttt_linear_bwd_workspace(const LinearBwdArgs& a, bool w0_shared);
cudaError_t launch_ttt_linear_bwd(LinearBwdArgs a, bool bf16, bool w0_shared, float* dW0, void* ws,
                                  cudaStream_t s);

}  // namespace ttt
