// LaCT SwiGLU fast-weight layer forward (placeholder until the kernels land).
#include "lact.cuh"

namespace ttt {

ttt_status lact_forward(const LactArgs&, cudaStream_t) { return TTT_ERR_UNSUPPORTED; }

}  // namespace ttt
