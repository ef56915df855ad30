// LaCT SwiGLU fast-weight layer: host-side interface of the chunk scan.
#pragma once

#include "common.cuh"

namespace ttt {

struct LactArgs {
  TokView q, k, v;
  EtaView eta;
  const float *W1, *W2, *W3;   // [H or B*H][dh][dk], [..][dv][dh], [..][dh][dk]
  int64_t w_sb[3];             // batch stride of W1, W2, W3 (0: shared over batch)
  TokViewMut out;
  float *W1_final, *W2_final, *W3_final;  // each may be null
  int B, H, T, dk, dv, dh, chunk, update_rule, causal, dtype;
  int* status;
  // Momentum update (lact_swiglu_fwd_momentum): M <- beta M + G, W <- W - M.
  int momentum;                // 0: GD / Muon as update_rule says
  float beta;
  const float* M0[3];          // initial momentum of W1, W2, W3 (null: zero)
  int64_t m0_sb[3];            // batch stride of M0 (0: shared over batch)
  float* M_final[3];           // each may be null
  // Context parallelism (lact_swiglu_fwd_cp): called once per chunk, after
  // the chunk's gradients are complete and before they are used, with the
  // contiguous fp32 gradient buffer (G1 | G3 | G2 of every (batch, head)).
  lact_grad_reduce_fn reduce;  // null: no exchange
  void* reduce_user;
};

// Enqueues the whole layer forward on `s`, taking its scratch from the
// device's default stream-ordered memory pool; returns a ttt_status.
ttt_status lact_forward(const LactArgs& a, cudaStream_t s);

// Bytes of device scratch lact_run needs for `a` (0 if `a` is unsupported).
size_t lact_scratch_bytes(const LactArgs& a);

// Same computation on caller-provided scratch of `bytes` >= lact_scratch_bytes(a),
// 256-byte aligned. Allocates nothing.
ttt_status lact_run(const LactArgs& a, cudaStream_t s, void* scratch, size_t bytes);

// Backward (lact_swiglu_bwd): upstream gradients in, gradients out.
struct LactBwdArgs {
  TokView dy;                         // [B,H,T,dv]
  const float *dW1_final, *dW2_final, *dW3_final;  // [B*H] x weight, each may be null
  TokViewMut dq, dk, dv;              // same element type as q
  float* deta;                        // [B,H,T] contiguous
  float *dW1, *dW2, *dW3;             // shape of W1, W2, W3 (batch-summed when shared)
};
bool lact_bwd_supported(const LactArgs& a);
// Enqueues the backward on `s` (fp32 arithmetic; allocates its workspace
// stream-ordered from the library's pool).
ttt_status lact_backward(const LactArgs& a, const LactBwdArgs& g, cudaStream_t s);

// Validates the C-ABI arguments of lact_swiglu_fwd_ex and fills `a`, except
// its status pointer. Makes no CUDA call.
ttt_status lact_build_args(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                           const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                           const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                           int32_t causal, const ttt_tensor* out, const ttt_tensor* W1_final,
                           const ttt_tensor* W2_final, const ttt_tensor* W3_final, LactArgs* a);

// Sets a->status to the current device's status word (TTT_ERR_CUDA if the
// device or the symbol cannot be queried).
ttt_status lact_attach_status(LactArgs* a);

}  // namespace ttt
