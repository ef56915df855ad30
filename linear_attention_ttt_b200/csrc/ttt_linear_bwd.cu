// TTT-Linear / inner-product layer backward (training): gradients of a scalar
// objective through the forward of ttt_linear_fwd, given dL/dy and dL/dW_final.
//
// The forward is the mini-batch GD rule of the "Test-Time Training (TTT)"
// summary ("병렬화: Mini-batch Gradient Descent"): in a chunk with start
// weights W_s, token t uses W_t = W_s - sum_{i<=t} eta_i g_i(W_s) and
// y_t = q_t W_t, with g_i = k_i^T e_i, e_i = k_i W_s - v_i (MSE, "예시 2") or
// g_i = -k_i^T v_i (inner product, "예시 1"); the chunk's last W_t starts the
// next chunk. Differentiating it token by token, with U_t = q_t^T dy_t and
// R_t = G + sum_{t' >= t in chunk} U_t' (G = dL/dW at the chunk end):
//   dq_t   = dy_t W_t^T
//   deta_t = -<R_t, g_t>
//   MSE:   de_t = -eta_t k_t R_t,  dk_t = -eta_t R_t e_t^T + de_t W_s^T,
//          dv_t = -de_t,           dL/dW_s = R_s + sum_t k_t^T de_t
//   inner product:  dk_t = eta_t R_t v_t^T,  dv_t = eta_t k_t R_t,
//          dL/dW_s = R_s
// and dL/dW_s becomes G of the previous chunk; after the first chunk it is
// dL/dW0.
//
// Layout: one CTA of 256 threads per (batch, head), fp32 arithmetic on the
// CUDA cores. A forward pass stores the start weights of every chunk (MSE)
// in a workspace, or only runs to the final weights (inner product, whose
// token gradients do not depend on W). The backward then walks the chunks in
// reverse and, inside each chunk, the tokens in reverse, carrying W_t
// (recovered from the chunk-end weights by adding each token's update back),
// R and the chunk's dL/dW_s contributions. Shared memory holds W_s, W_t and
// R; the per-thread part of sum_t k_t^T de_t stays in registers.
#include "common.cuh"

namespace ttt {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxElems = 128 * 128;                  // dk * dv
constexpr int kRegs = kMaxElems / kThreads;           // per-thread dW_s part

template <typename T>
__device__ __forceinline__ float ld(const TokView& v, int b, int h, int64_t t, int c) {
  return to_f32((static_cast<const T*>(v.p) + b * v.sb + h * v.sh + t * v.st)[c]);
}
template <typename T>
__device__ __forceinline__ void st(const TokViewMut& v, int b, int h, int64_t t, int c, float x) {
  (static_cast<T*>(v.p) + b * v.sb + h * v.sh + t * v.st)[c] = T(x);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) ttt_linear_bwd_kernel(LinearBwdArgs a) {
  extern __shared__ float smem[];
  const int dk = a.dk, dv = a.dv, n = dk * dv;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int tid = threadIdx.x;
  const bool mse = a.loss == TTT_LOSS_MSE;

  float* Ws = smem;            // [dk][dv] chunk-start weights
  float* Wt = Ws + n;          // [dk][dv] weights after the current token
  float* R = Wt + n;           // [dk][dv]
  float* qv = R + n;           // [dk]
  float* kv = qv + dk;         // [dk]
  float* vv = kv + dk;         // [dv]
  float* dyv = vv + dv;        // [dv]
  float* ev = dyv + dv;        // [dv] e_t (MSE) or v_t (inner product)
  float* kR = ev + dv;         // [dv]
  float* Rx = kR + dv;         // [dk] R_t e_t^T or R_t v_t^T
  float* red = Rx + dk;        // [8] warp partials
  float* etas = red + 8;       // [1]

  const float* eta = a.eta.p + b * a.eta.sb + h * a.eta.sh;
  auto load_tok = [&](int t, bool with_q) {
    for (int c = tid; c < dk; c += kThreads) {
      kv[c] = ld<T>(a.k, b, h, t, c);
      if (with_q) qv[c] = ld<T>(a.q, b, h, t, c);
    }
    for (int c = tid; c < dv; c += kThreads) {
      vv[c] = ld<T>(a.v, b, h, t, c);
      if (with_q) dyv[c] = ld<T>(a.dy, b, h, t, c);
    }
    if (tid == 0) etas[0] = eta[(int64_t)t * a.eta.st];
  };
  // ev = k W_s - v (MSE) or v (inner product), one thread per column
  auto make_e = [&]() {
    for (int c = tid; c < dv; c += kThreads) {
      if (mse) {
        float acc = 0.f;
        for (int r = 0; r < dk; ++r) acc = fmaf(kv[r], Ws[r * dv + c], acc);
        ev[c] = acc - vv[c];
      } else {
        ev[c] = vv[c];
      }
    }
  };

  // ---- forward: chunk-start weights (MSE) and the final weights ----
  const float* W0 = a.W0 + b * a.w0_sb + (int64_t)h * n;
  for (int x = tid; x < n; x += kThreads) Ws[x] = Wt[x] = W0[x];
  __syncthreads();
  float* ck = a.ckpt ? a.ckpt + (int64_t)bh * a.nchunks * n : nullptr;
  for (int c = 0; c < a.nchunks; ++c) {
    const int s0 = c * a.chunk, e0 = min(s0 + a.chunk, a.T);
    if (mse)
      for (int x = tid; x < n; x += kThreads) ck[(int64_t)c * n + x] = Ws[x];
    for (int t = s0; t < e0; ++t) {
      load_tok(t, false);
      __syncthreads();
      make_e();
      __syncthreads();
      // W_t = W_{t-1} - eta_t k_t^T e_t (MSE) or + eta_t k_t^T v_t
      const float sc = mse ? -etas[0] : etas[0];
      for (int x = tid; x < n; x += kThreads) Wt[x] = fmaf(sc * kv[x / dv], ev[x % dv], Wt[x]);
      __syncthreads();
    }
    for (int x = tid; x < n; x += kThreads) Ws[x] = Wt[x];
    __syncthreads();
  }
  // Wt = W_final now.

  // ---- backward ----
  const float* G0 = a.dWf ? a.dWf + (int64_t)bh * n : nullptr;
  for (int x = tid; x < n; x += kThreads) R[x] = G0 ? G0[x] : 0.f;
  float acc[kRegs];
#pragma unroll
  for (int i = 0; i < kRegs; ++i) acc[i] = 0.f;
  float* dq_eta = a.deta + (int64_t)bh * a.T;
  for (int c = a.nchunks - 1; c >= 0; --c) {
    const int s0 = c * a.chunk, e0 = min(s0 + a.chunk, a.T);
    if (mse)
      for (int x = tid; x < n; x += kThreads) Ws[x] = ck[(int64_t)c * n + x];
    __syncthreads();
    for (int t = e0 - 1; t >= s0; --t) {
      load_tok(t, true);
      __syncthreads();
      make_e();
      // dq_t = dy_t W_t^T (reads shared memory only, like make_e)
      for (int r = tid; r < dk; r += kThreads) {
        float s = 0.f;
        for (int j = 0; j < dv; ++j) s = fmaf(dyv[j], Wt[r * dv + j], s);
        st<T>(a.gq, b, h, t, r, s);
      }
      __syncthreads();
      // R += q_t^T dy_t; W_{t-1} = W_t + eta_t k_t^T e_t (MSE) or - eta_t k_t^T v_t
      const float et = etas[0];
      const float sc = mse ? et : -et;
      for (int x = tid; x < n; x += kThreads) {
        const int r = x / dv, j = x % dv;
        R[x] = fmaf(qv[r], dyv[j], R[x]);
        Wt[x] = fmaf(sc * kv[r], ev[j], Wt[x]);
      }
      __syncthreads();
      // kR = k_t R_t (per column), Rx = R_t e_t^T (per row)
      for (int j = tid; j < dv; j += kThreads) {
        float s = 0.f;
        for (int r = 0; r < dk; ++r) s = fmaf(kv[r], R[r * dv + j], s);
        kR[j] = s;
      }
      for (int r = tid; r < dk; r += kThreads) {
        float s = 0.f;
        for (int j = 0; j < dv; ++j) s = fmaf(R[r * dv + j], ev[j], s);
        Rx[r] = s;
      }
      __syncthreads();
      // deta_t = -<R_t, g_t>: MSE -(k R) . e, inner product (k R) . v
      {
        float p = 0.f;
        for (int j = tid; j < dv; j += kThreads) p = fmaf(kR[j], ev[j], p);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
        if ((tid & 31) == 0) red[tid >> 5] = p;
      }
      __syncthreads();
      if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) s += red[w];
        dq_eta[t] = mse ? -s : s;
      }
      // dv_t and (MSE) de_t = -dv_t, kept in kR
      for (int j = tid; j < dv; j += kThreads) {
        const float dvj = et * kR[j];
        st<T>(a.gv, b, h, t, j, dvj);
        kR[j] = -dvj;
      }
      __syncthreads();
      // dk_t; MSE: dL/dW_s += k_t^T de_t
      for (int r = tid; r < dk; r += kThreads) {
        float s;
        if (mse) {
          s = -et * Rx[r];
          for (int j = 0; j < dv; ++j) s = fmaf(kR[j], Ws[r * dv + j], s);
        } else {
          s = et * Rx[r];
        }
        st<T>(a.gk, b, h, t, r, s);
      }
      if (mse) {
#pragma unroll
        for (int i = 0; i < kRegs; ++i) {
          const int x = tid + i * kThreads;
          if (x < n) acc[i] = fmaf(kv[x / dv], kR[x % dv], acc[i]);
        }
      }
      __syncthreads();
    }
    // chunk start: G = R + sum_t k_t^T de_t carries into the previous chunk,
    // whose end weights are this chunk's start weights
#pragma unroll
    for (int i = 0; i < kRegs; ++i) {
      const int x = tid + i * kThreads;
      if (x < n) {
        R[x] += acc[i];
        acc[i] = 0.f;
      }
    }
    if (mse)
      for (int x = tid; x < n; x += kThreads) Wt[x] = Ws[x];
    __syncthreads();
  }
  float* dW = a.dW + (int64_t)bh * n;
  for (int x = tid; x < n; x += kThreads) dW[x] = R[x];
}

// dL/dW0 of a weight shared over the batch: the sum over b in a fixed order.
__global__ void sum_over_batch_kernel(float* dst, const float* src, int B, int64_t per_b) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < per_b;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += src[(int64_t)b * per_b + i];
    dst[i] = s;
  }
}

}  // namespace

bool ttt_linear_bwd_supported(int dk, int dv) { return dk <= 128 && dv <= 128 && dk * dv <= kMaxElems; }

size_t ttt_linear_bwd_workspace(const LinearBwdArgs& a, bool w0_shared) {
  const int64_t n = (int64_t)a.dk * a.dv, Z = (int64_t)a.B * a.H;
  size_t f = 0;
  if (a.loss == TTT_LOSS_MSE) f += (size_t)(Z * a.nchunks * n);
  if (w0_shared) f += (size_t)(Z * n);
  return f * sizeof(float);
}

// `ws` holds ttt_linear_bwd_workspace() bytes; dW0 is [H,dk,dv] when
// w0_shared (summed over the batch) and [B,H,dk,dv] otherwise.
cudaError_t launch_ttt_linear_bwd(LinearBwdArgs a, bool bf16, bool w0_shared, float* dW0, void* ws,
                                  cudaStream_t s) {
  const int64_t n = (int64_t)a.dk * a.dv, Z = (int64_t)a.B * a.H;
  float* f = static_cast<float*>(ws);
  a.ckpt = nullptr;
  if (a.loss == TTT_LOSS_MSE) {
    a.ckpt = f;
    f += Z * a.nchunks * n;
  }
  a.dW = w0_shared ? f : dW0;
  const size_t smem = sizeof(float) * (3 * n + 3 * a.dk + 4 * a.dv + 9);
  cudaError_t e;
  if (bf16) {
    e = cudaFuncSetAttribute(ttt_linear_bwd_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ttt_linear_bwd_kernel<__nv_bfloat16><<<(int)Z, kThreads, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(ttt_linear_bwd_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ttt_linear_bwd_kernel<float><<<(int)Z, kThreads, smem, s>>>(a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (w0_shared) {
    const int64_t per_b = (int64_t)a.H * n;
    const int blocks = (int)((per_b + 255) / 256 < 1184 ? (per_b + 255) / 256 : 1184);
    sum_over_batch_kernel<<<blocks, 256, 0, s>>>(dW0, a.dW, a.B, per_b);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace ttt
