// TTT-Linear / inner-product layer forward for bf16 tokens (placeholder).
#include "common.cuh"

namespace ttt {

cudaError_t launch_ttt_linear_bf16(const LinearArgs&, cudaStream_t, bool* supported) {
  *supported = false;
  return cudaSuccess;
}

}  // namespace ttt
