// TTT-Linear / inner-product layer forward on the CUDA cores with fp32
// arithmetic throughout: every fp32 shape, and the bf16 head sizes the
// tensor-core kernels do not cover (dk or dv other than 64 / 128, dk != dv).
//
// Computes, per (batch, head), the mini-batch GD rule of the "Test-Time
// Training (TTT)" summary ("병렬화: Mini-batch Gradient Descent"): with t' the
// chunk start,  y_t = q_t W_t,  W_t = W_{t'} - sum_{i=t'}^{t} eta_i k_i^T e_i,
// e_i = k_i W_{t'} - v_i (MSE, "예시 2") or e_i = -v_i (inner product,
// "예시 1"). It walks a chunk in blocks of 16 tokens and keeps two fp32
// matrices in shared memory: the chunk-start weights W_{t'} and the running
// sum dW of the chunk's updates so far, so that for a token t in the current
// block
//   y_t = q_t (W_{t'} - dW) - sum_{i in block, i <= t} eta_i (q_t . k_i) e_i.
// Any chunk size works, including a shorter last chunk.
//
// Grid: (B*H, ceil(dv/32)); each CTA owns 32 output columns of one head. The
// columns of W are independent in this rule, so no CTA talks to another.
// The next block's tokens are fetched into registers while the current block
// is computed, so that each block waits for at most one round of loads.
#include "common.cuh"

namespace ttt {
namespace {

constexpr int kCols = 32;     // W columns per CTA
constexpr int kTB = 16;       // tokens per block
constexpr int kThreads = 256;
constexpr int kMaxDk = 256;                        // the entry points reject larger heads
constexpr int kQK = kTB * kMaxDk / kThreads;       // q and k values per thread and block
constexpr int kV = kTB * kCols / kThreads;         // v values per thread and block
static_assert(kV * kThreads == kTB * kCols, "v block split");

template <typename T>
__device__ __forceinline__ const T* tok_row(const TokView& v, int b, int h, int64_t t) {
  return static_cast<const T*>(v.p) + b * v.sb + h * v.sh + t * v.st;
}

template <typename TT>
__global__ void __launch_bounds__(kThreads, 2)
ttt_linear_f32_kernel(LinearArgs a) {
  extern __shared__ float smem[];
  const int dk = a.dk, dv = a.dv;
  const int bh = blockIdx.x;
  const int b = bh / a.H, h = bh % a.H;
  const int j0 = blockIdx.y * kCols;
  const int ncol = min(kCols, dv - j0);
  const int tid = threadIdx.x;

  float* Wst = smem;                 // [dk][kCols] chunk-start weights
  float* dW = Wst + dk * kCols;      // [dk][kCols] sum of this chunk's updates
  float* Qs = dW + dk * kCols;       // [kTB][dk]
  float* Ks = Qs + kTB * dk;         // [kTB][dk]
  float* Vs = Ks + kTB * dk;         // [kTB][kCols]
  float* Es = Vs + kTB * kCols;      // [kTB][kCols]
  float* Ss = Es + kTB * kCols;      // [kTB][kTB]  q_t . k_i
  float* etas = Ss + kTB * kTB;      // [kTB]

  const float* W0 = a.W0 + b * a.w0_sb + (int64_t)h * dk * dv;
  for (int x = tid; x < dk * kCols; x += kThreads) {
    int r = x / kCols, c = x % kCols;
    Wst[x] = (c < ncol) ? W0[(int64_t)r * dv + j0 + c] : 0.f;
    dW[x] = 0.f;
  }
  __syncthreads();

  const float* eta = a.eta.p + b * a.eta.sb + h * a.eta.sh;
  if (!TTT_BOUNDS(dk <= kMaxDk && a.chunk > 0, a.status)) return;
  // the block of tokens after the one at t0 (blocks never cross a chunk end)
  auto block_len = [&](int t0) {
    const int ce = min((t0 / a.chunk) * a.chunk + a.chunk, a.T);
    return min(kTB, ce - t0);
  };
  float pq[kQK], pk[kQK], pv[kV], pe = 0.f;
  auto fetch = [&](int t0, int nt) {
#pragma unroll
    for (int j = 0; j < kQK; ++j) {
      const int x = tid + j * kThreads;
      const int i = x / dk, c = x % dk;
      const bool ok = x < kTB * dk && i < nt;
      pq[j] = ok ? to_f32(tok_row<TT>(a.q, b, h, t0 + i)[c]) : 0.f;
      pk[j] = ok ? to_f32(tok_row<TT>(a.k, b, h, t0 + i)[c]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      const int x = tid + j * kThreads;
      const int i = x / kCols, c = x % kCols;
      pv[j] = (i < nt && c < ncol) ? to_f32(tok_row<TT>(a.v, b, h, t0 + i)[j0 + c]) : 0.f;
    }
    if (tid < kTB) pe = tid < nt ? eta[(int64_t)(t0 + tid) * a.eta.st] : 0.f;
  };
  if (a.T > 0) fetch(0, block_len(0));
  for (int cs = 0; cs < a.T; cs += a.chunk) {
    const int ce = min(cs + a.chunk, a.T);
    for (int t0 = cs; t0 < ce; t0 += kTB) {
      const int nt = min(kTB, ce - t0);
      // the previous block's last barrier has passed: the staging buffers are free
#pragma unroll
      for (int j = 0; j < kQK; ++j) {
        const int x = tid + j * kThreads;
        if (x < kTB * dk) Qs[x] = pq[j], Ks[x] = pk[j];
      }
#pragma unroll
      for (int j = 0; j < kV; ++j) Vs[tid + j * kThreads] = pv[j];
      if (tid < kTB) etas[tid] = pe;
      if (t0 + nt < a.T) fetch(t0 + nt, block_len(t0 + nt));
      __syncthreads();

      // e_i at the chunk-start weights; scores q_t . k_i. Each thread owns
      // kV outputs whose sums run side by side (each in its own fixed order).
      {
        float acc[kV] = {};
        if (a.loss == TTT_LOSS_MSE) {
#pragma unroll 4
          for (int r = 0; r < dk; ++r) {
#pragma unroll
            for (int j = 0; j < kV; ++j) {
              const int x = tid + j * kThreads;
              acc[j] = fmaf(Ks[(x / kCols) * dk + r], Wst[r * kCols + x % kCols], acc[j]);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kV; ++j) Es[tid + j * kThreads] = acc[j] - Vs[tid + j * kThreads];
      }
      if (tid < kTB * kTB) {
        int t = tid / kTB, i = tid % kTB;
        float acc = 0.f;
        if (i <= t) {
#pragma unroll 4
          for (int r = 0; r < dk; ++r) acc = fmaf(Qs[t * dk + r], Ks[i * dk + r], acc);
        }
        Ss[tid] = acc;
      }
      __syncthreads();

      // y_t = q_t (W_{t'} - dW) - sum_{i<=t} eta_i s_ti e_i
      {
        float acc[kV] = {};
#pragma unroll 4
        for (int r = 0; r < dk; ++r) {
#pragma unroll
          for (int j = 0; j < kV; ++j) {
            const int x = tid + j * kThreads, t = x / kCols, c = x % kCols;
            acc[j] = fmaf(Qs[t * dk + r], Wst[r * kCols + c] - dW[r * kCols + c], acc[j]);
          }
        }
#pragma unroll
        for (int j = 0; j < kV; ++j) {
          const int x = tid + j * kThreads, t = x / kCols, c = x % kCols;
          if (t < nt && c < ncol) {
            for (int i = 0; i <= t; ++i)
              acc[j] = fmaf(-etas[i] * Ss[t * kTB + i], Es[i * kCols + c], acc[j]);
            TT* o = static_cast<TT*>(a.out.p) + b * a.out.sb + h * a.out.sh +
                    (int64_t)(t0 + t) * a.out.st;
            o[j0 + c] = TT(acc[j]);
          }
        }
      }
      __syncthreads();

      // dW += sum_i eta_i k_i^T e_i: thread (r0 = tid / kCols, c = tid % kCols)
      // owns rows r0, r0 + 8, ..., eight of them at a time
      {
        constexpr int kRowStep = kThreads / kCols, kU = 8;
        const int c = tid % kCols, r0 = tid / kCols;
        for (int rb = 0; rb < dk; rb += kU * kRowStep) {
          float acc[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int r = rb + r0 + u * kRowStep;
            acc[u] = r < dk ? dW[r * kCols + c] : 0.f;
          }
          for (int i = 0; i < nt; ++i) {
            const float e = Es[i * kCols + c];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
              const int r = rb + r0 + u * kRowStep;
              if (r < dk) acc[u] = fmaf(etas[i] * Ks[i * dk + r], e, acc[u]);
            }
          }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int r = rb + r0 + u * kRowStep;
            if (r < dk) dW[r * kCols + c] = acc[u];
          }
        }
      }
      __syncthreads();
    }
    for (int x = tid; x < dk * kCols; x += kThreads) {
      Wst[x] -= dW[x];
      dW[x] = 0.f;
    }
    __syncthreads();
  }

  if (a.W_final) {
    float* Wf = a.W_final + (int64_t)bh * dk * dv;
    for (int x = tid; x < dk * kCols; x += kThreads) {
      int r = x / kCols, c = x % kCols;
      if (c < ncol) Wf[(int64_t)r * dv + j0 + c] = Wst[x];
    }
  }
}

template <typename TT>
cudaError_t launch_cc(const LinearArgs& a, cudaStream_t s) {
  const size_t smem =
      sizeof(float) * (2 * a.dk * kCols + 2 * kTB * a.dk + 2 * kTB * kCols + kTB * kTB + kTB);
  cudaError_t e = cudaFuncSetAttribute(ttt_linear_f32_kernel<TT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.B * a.H, (a.dv + kCols - 1) / kCols);
  ttt_linear_f32_kernel<TT><<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ttt_linear_f32(const LinearArgs& a, cudaStream_t s) {
  return launch_cc<float>(a, s);
}

cudaError_t launch_ttt_linear_cc_bf16(const LinearArgs& a, cudaStream_t s) {
  return launch_cc<__nv_bfloat16>(a, s);
}

}  // namespace ttt
