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
};

// Enqueues the whole layer forward on `s`; returns a ttt_status.
ttt_status lact_forward(const LactArgs& a, cudaStream_t s);

}  // namespace ttt
