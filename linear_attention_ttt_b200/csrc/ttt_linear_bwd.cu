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
// In matrix form over a chunk (rows = tokens, N = diag(eta), E the rows e_t,
// masks inclusive of the diagonal) these are
//   dQ = dY W_s^T - tril(dY E^T) N K,
//   kR = K G + triu(K Q^T) dY,   Rx = E G^T + triu(E dY^T) Q   (rows k_t R_t, R_t e_t^T),
//   dL/dW_s = G + Q^T dY (+ K^T dE for MSE),
// so only G links one chunk to the one before it.
//
// Layout: one CTA of 256 (heads up to 64) or 512 threads per (batch, head), fp32 arithmetic on the
// CUDA cores, 16-token blocks staged in shared memory. Pass 1 walks the
// chunks forward: it stores the chunk-start weights (MSE) in a workspace and
// computes dQ with the running sum of the chunk's updates. Pass 2 walks the
// chunks, and the blocks inside each chunk, in reverse, carrying R (G plus
// the q^T dy of the later tokens of the chunk) in shared memory and the
// chunk's sum_t k_t^T de_t in registers. Weight-shaped arrays in shared
// memory have a row stride of dv + 1 floats and token tiles of d + 1, so that
// walks along either index are free of bank conflicts.
#include "common.cuh"

namespace ttt {
namespace {

// threads per CTA: 256 for heads up to 64, 512 for heads up to 128 (so that
// the per-thread register arrays stay at 16-32 elements)
__host__ __device__ constexpr int threads_for(int D) { return D == 128 ? 512 : 256; }
constexpr int kTB = 16;                                // tokens per block
constexpr int kMaxD = 128;                             // dk, dv <= 128
constexpr int kLdS = kTB + 1;                          // row stride of the 16 x 16 tiles

template <typename T>
__device__ __forceinline__ float ld(const TokView& v, int b, int h, int64_t t, int c) {
  return to_f32((static_cast<const T*>(v.p) + b * v.sb + h * v.sh + t * v.st)[c]);
}
template <typename T>
__device__ __forceinline__ void st(const TokViewMut& v, int b, int h, int64_t t, int c, float x) {
  (static_cast<T*>(v.p) + b * v.sb + h * v.sh + t * v.st)[c] = T(x);
}

// 4-byte asynchronous copy global -> shared (no register round trip)
__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
// waits for this thread's copies; a barrier after it publishes them to the CTA
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

__host__ __device__ constexpr size_t bwd_smem_floats(int dk, int dv) {
  return 2 * (size_t)dk * (dv + 1) + 3 * (size_t)kTB * (dk + 1) + 4 * (size_t)kTB * (dv + 1) +
         2 * kTB * kLdS + kTB;
}

// kDiv: dk and dv divide the thread count, so that the element a thread owns
// in pass u of a flat walk keeps its column: (tid + u * kNT) % d = tid % d.
// The index helpers then give the same elements with a column the compiler
// sees as fixed, and loads along that column are shared across the passes.
// D: the largest dk, dv the instance takes (64 or 128); it sizes the
// per-thread register arrays, so that small heads run a smaller body.
template <typename T, bool kDiv, int D>
__global__ void __launch_bounds__(threads_for(D), 1) ttt_linear_bwd_kernel(LinearBwdArgs a) {
  constexpr int kNT = threads_for(D);
  constexpr int kRegs = D * D / kNT;   // weight elements per thread
  constexpr int kOut = kTB * D / kNT;  // token-tile elements per thread
  extern __shared__ float smem[];
  const int dk = a.dk, dv = a.dv, n = dk * dv;
  const int ldw = dv + 1, ldk = dk + 1, ldv = dv + 1;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool mse = a.loss == TTT_LOSS_MSE;
  if (!TTT_BOUNDS(dk <= D && dv <= D && a.chunk > 0 &&
                      (!kDiv || (kNT % dk == 0 && kNT % dv == 0)),
                  a.status))
    return;
  // row and column of element tid + u * kNT of a flat [.][d] walk
  auto row_of = [&](int u, int d) {
    return kDiv ? tid / d + (kNT / d) * u : (tid + u * kNT) / d;
  };
  auto col_of = [&](int u, int d) { return kDiv ? tid % d : (tid + u * kNT) % d; };

  float* Ws = smem;              // [dk][ldw] chunk-start weights
  float* Acc = Ws + dk * ldw;    // [dk][ldw] pass 1: the chunk's updates so far; pass 2: R
  float* Qs = Acc + dk * ldw;    // [kTB][ldk]
  float* Ks = Qs + kTB * ldk;    // [kTB][ldk]
  float* Zs = Ks + kTB * ldk;    // [kTB][ldk]  R_t e_t^T
  float* Vs = Zs + kTB * ldk;    // [kTB][ldv]  v, then de (pass 2)
  float* Ys = Vs + kTB * ldv;    // [kTB][ldv]  dy
  float* Es = Ys + kTB * ldv;    // [kTB][ldv]  e
  float* Xs = Es + kTB * ldv;    // [kTB][ldv]  k_t R_t
  float* S1 = Xs + kTB * ldv;    // [kTB][kLdS]
  float* S2 = S1 + kTB * kLdS;   // [kTB][kLdS]
  float* etas = S2 + kTB * kLdS; // [kTB]

  const float* eta = a.eta.p + b * a.eta.sb + h * a.eta.sh;
  // tokens [t0, t0 + nt) into the tiles, zero rows after nt: every load is
  // issued before the first shared-memory store, so that the block waits for
  // one round trip
  auto load_block = [&](int t0, int nt) {
    float qv[kOut], kv[kOut], vv[kOut], yv[kOut];
#pragma unroll
    for (int u = 0; u < kOut; ++u) {
      const int t = row_of(u, dk), r = col_of(u, dk);
      const bool ok = t < kTB && t < nt;
      qv[u] = ok ? ld<T>(a.q, b, h, t0 + t, r) : 0.f;
      kv[u] = ok ? ld<T>(a.k, b, h, t0 + t, r) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kOut; ++u) {
      const int t = row_of(u, dv), j = col_of(u, dv);
      const bool ok = t < kTB && t < nt;
      vv[u] = ok ? ld<T>(a.v, b, h, t0 + t, j) : 0.f;
      yv[u] = ok ? ld<T>(a.dy, b, h, t0 + t, j) : 0.f;
    }
    const float ev = tid < nt ? eta[(int64_t)(t0 + tid) * a.eta.st] : 0.f;
#pragma unroll
    for (int u = 0; u < kOut; ++u) {
      const int t = row_of(u, dk), r = col_of(u, dk);
      if (t < kTB) Qs[t * ldk + r] = qv[u], Ks[t * ldk + r] = kv[u];
    }
#pragma unroll
    for (int u = 0; u < kOut; ++u) {
      const int t = row_of(u, dv), j = col_of(u, dv);
      if (t < kTB) Vs[t * ldv + j] = vv[u], Ys[t * ldv + j] = yv[u];
    }
    if (tid < kTB) etas[tid] = ev;
  };
  // a dense [dk][dv] fp32 matrix into a weight-shaped array (asynchronous;
  // cp_async_wait_all and a barrier before use)
  auto fetch_weights = [&](float* dst, const float* src) {
    for (int x = tid; x < n; x += kNT) cp_async4(dst + (x / dv) * ldw + x % dv, src + x);
  };
  // E = K W_s - V (MSE) or -V (inner product)
  auto make_e = [&]() {
    float acc[kOut];
    int ti[kOut], ji[kOut];
#pragma unroll
    for (int u = 0; u < kOut; ++u) {
      ti[u] = row_of(u, dv), ji[u] = col_of(u, dv), acc[u] = 0.f;
    }
    if (mse) {
#pragma unroll 4
      for (int r = 0; r < dk; ++r) {
#pragma unroll
        for (int u = 0; u < kOut; ++u)
          if (ti[u] < kTB) acc[u] = fmaf(Ks[ti[u] * ldk + r], Ws[r * ldw + ji[u]], acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kOut; ++u)
      if (ti[u] < kTB) Es[ti[u] * ldv + ji[u]] = acc[u] - Vs[ti[u] * ldv + ji[u]];
  };

  // ---- pass 1: chunk-start weights (MSE) and dQ ----
  const float* W0 = a.W0 + b * a.w0_sb + (int64_t)h * n;
  fetch_weights(Ws, W0);
  cp_async_wait_all();
  float* ck = a.ckpt ? a.ckpt + (int64_t)bh * a.nchunks * n : nullptr;
  for (int c = 0; c < a.nchunks; ++c) {
    const int s0 = c * a.chunk, e0 = min(s0 + a.chunk, a.T);
    for (int x = tid; x < n; x += kNT) {
      const int r = x / dv, j = x % dv;
      if (mse) ck[(int64_t)c * n + x] = Ws[r * ldw + j];
      Acc[r * ldw + j] = 0.f;
    }
    for (int t0 = s0; t0 < e0; t0 += kTB) {
      const int nt = min(kTB, e0 - t0);
      __syncthreads();  // the previous block is done with the tiles
      load_block(t0, nt);
      __syncthreads();
      make_e();
      __syncthreads();
      // S1[t][i] = eta_i (dy_t . e_i) for i <= t
      if (tid < kTB * kTB) {
        const int t = tid / kTB, i = tid % kTB;
        float acc = 0.f;
        if (i <= t && t < nt) {
#pragma unroll 4
          for (int j = 0; j < dv; ++j) acc = fmaf(Ys[t * ldv + j], Es[i * ldv + j], acc);
        }
        S1[t * kLdS + i] = etas[i] * acc;
      }
      __syncthreads();
      // dq_t = dy_t (W_s - Acc)^T - sum_{i <= t} S1[t][i] k_i
      {
        float acc[kOut];
        int ti[kOut], ri[kOut];
#pragma unroll
        for (int u = 0; u < kOut; ++u) {
          ti[u] = row_of(u, dk), ri[u] = col_of(u, dk), acc[u] = 0.f;
        }
#pragma unroll 4
        for (int j = 0; j < dv; ++j) {
#pragma unroll
          for (int u = 0; u < kOut; ++u)
            if (ti[u] < kTB)
              acc[u] = fmaf(Ys[ti[u] * ldv + j], Ws[ri[u] * ldw + j] - Acc[ri[u] * ldw + j], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < kOut; ++u) {
          if (ti[u] >= nt) continue;
          for (int i = 0; i <= ti[u]; ++i)
            acc[u] = fmaf(-S1[ti[u] * kLdS + i], Ks[i * ldk + ri[u]], acc[u]);
          st<T>(a.gq, b, h, t0 + ti[u], ri[u], acc[u]);
        }
      }
      __syncthreads();
      // Acc += K^T N E
      for (int x0 = 0; x0 < n; x0 += 8 * kNT) {
        float acc[8];
        int ri[8], ji[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          ri[u] = row_of(x0 / kNT + u, dv), ji[u] = col_of(x0 / kNT + u, dv);
          acc[u] = ri[u] < dk ? Acc[ri[u] * ldw + ji[u]] : 0.f;
        }
        for (int i = 0; i < nt; ++i) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (ri[u] < dk) acc[u] = fmaf(etas[i] * Ks[i * ldk + ri[u]], Es[i * ldv + ji[u]], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (ri[u] < dk) Acc[ri[u] * ldw + ji[u]] = acc[u];
      }
    }
    __syncthreads();
    for (int x = tid; x < n; x += kNT) {
      const int r = x / dv, j = x % dv;
      Ws[r * ldw + j] -= Acc[r * ldw + j];
    }
    __syncthreads();
  }

  // ---- pass 2: reverse ----
  const float* G0 = a.dWf ? a.dWf + (int64_t)bh * n : nullptr;
  if (G0) {
    fetch_weights(Acc, G0);
    cp_async_wait_all();
  } else {
    for (int x = tid; x < n; x += kNT) Acc[(x / dv) * ldw + x % dv] = 0.f;
  }
  float kde[kRegs];  // this thread's part of sum_t k_t^T de_t over the chunk
#pragma unroll
  for (int u = 0; u < kRegs; ++u) kde[u] = 0.f;
  float* deta_out = a.deta + (int64_t)bh * a.T;
  for (int c = a.nchunks - 1; c >= 0; --c) {
    const int s0 = c * a.chunk, e0 = min(s0 + a.chunk, a.T);
    __syncthreads();  // every thread is done with the later chunk's weights
    if (mse) fetch_weights(Ws, ck + (int64_t)c * n);  // waited for below, with the tokens
    const int nb = (e0 - s0 + kTB - 1) / kTB;
    for (int bi = nb - 1; bi >= 0; --bi) {
      const int t0 = s0 + bi * kTB, nt = min(kTB, e0 - t0);
      __syncthreads();  // the previous block is done with the tiles
      load_block(t0, nt);
      cp_async_wait_all();  // the chunk's weights, at its first block
      __syncthreads();
      make_e();
      // S1[t][t'] = k_t . q_t' for t <= t'
      if (tid < kTB * kTB) {
        const int t = tid / kTB, tp = tid % kTB;
        float acc = 0.f;
        if (t <= tp && tp < nt) {
#pragma unroll 4
          for (int r = 0; r < dk; ++r) acc = fmaf(Ks[t * ldk + r], Qs[tp * ldk + r], acc);
        }
        S1[t * kLdS + tp] = acc;
      }
      __syncthreads();
      // S2[t][t'] = e_t . dy_t' for t <= t'
      if (tid < kTB * kTB) {
        const int t = tid / kTB, tp = tid % kTB;
        float acc = 0.f;
        if (t <= tp && tp < nt) {
#pragma unroll 4
          for (int j = 0; j < dv; ++j) acc = fmaf(Es[t * ldv + j], Ys[tp * ldv + j], acc);
        }
        S2[t * kLdS + tp] = acc;
      }
      __syncthreads();
      // kR = K R + S1 dY,  Rx = E R^T + S2 Q
      {
        float acc[kOut];
        int ti[kOut], ji[kOut];
#pragma unroll
        for (int u = 0; u < kOut; ++u) {
          ti[u] = row_of(u, dv), ji[u] = col_of(u, dv), acc[u] = 0.f;
        }
#pragma unroll 4
        for (int r = 0; r < dk; ++r) {
#pragma unroll
          for (int u = 0; u < kOut; ++u)
            if (ti[u] < kTB) acc[u] = fmaf(Ks[ti[u] * ldk + r], Acc[r * ldw + ji[u]], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < kOut; ++u) {
          if (ti[u] >= kTB) continue;
          for (int tp = ti[u]; tp < kTB; ++tp)
            acc[u] = fmaf(S1[ti[u] * kLdS + tp], Ys[tp * ldv + ji[u]], acc[u]);
          Xs[ti[u] * ldv + ji[u]] = acc[u];
        }
      }
      {
        float acc[kOut];
        int ti[kOut], ri[kOut];
#pragma unroll
        for (int u = 0; u < kOut; ++u) {
          ti[u] = row_of(u, dk), ri[u] = col_of(u, dk), acc[u] = 0.f;
        }
#pragma unroll 4
        for (int j = 0; j < dv; ++j) {
#pragma unroll
          for (int u = 0; u < kOut; ++u)
            if (ti[u] < kTB) acc[u] = fmaf(Es[ti[u] * ldv + j], Acc[ri[u] * ldw + j], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < kOut; ++u) {
          if (ti[u] >= kTB) continue;
          for (int tp = ti[u]; tp < kTB; ++tp)
            acc[u] = fmaf(S2[ti[u] * kLdS + tp], Qs[tp * ldk + ri[u]], acc[u]);
          Zs[ti[u] * ldk + ri[u]] = acc[u];
        }
      }
      __syncthreads();
      // deta_t = -(k_t R_t) . e_t; dv_t = eta_t k_t R_t; de_t = -dv_t (into Vs)
      for (int t = warp; t < kTB; t += kNT / 32) {
        float p = 0.f;
        for (int j = lane; j < dv; j += 32) p = fmaf(Xs[t * ldv + j], Es[t * ldv + j], p);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
        if (lane == 0 && t < nt) deta_out[t0 + t] = -p;
      }
#pragma unroll
      for (int u = 0; u < kOut; ++u) {
        const int t = row_of(u, dv), j = col_of(u, dv);
        if (t < kTB) {
          const float dvj = etas[t] * Xs[t * ldv + j];
          if (t < nt) st<T>(a.gv, b, h, t0 + t, j, dvj);
          Vs[t * ldv + j] = -dvj;
        }
      }
      __syncthreads();
      // dk_t = -eta_t R_t e_t^T (+ de_t W_s^T for MSE)
      {
        float acc[kOut];
        int ti[kOut], ri[kOut];
#pragma unroll
        for (int u = 0; u < kOut; ++u) {
          ti[u] = row_of(u, dk), ri[u] = col_of(u, dk), acc[u] = 0.f;
        }
        if (mse) {
#pragma unroll 4
          for (int j = 0; j < dv; ++j) {
#pragma unroll
            for (int u = 0; u < kOut; ++u)
              if (ti[u] < kTB) acc[u] = fmaf(Vs[ti[u] * ldv + j], Ws[ri[u] * ldw + j], acc[u]);
          }
        }
#pragma unroll
        for (int u = 0; u < kOut; ++u)
          if (ti[u] < nt)
            st<T>(a.gk, b, h, t0 + ti[u], ri[u],
                  acc[u] - etas[ti[u]] * Zs[ti[u] * ldk + ri[u]]);
      }
      // R += Q^T dY (R is read above only before the last barrier);
      // MSE: the chunk's sum_t k_t^T de_t
      {
        float yc[kTB], dc[kTB];  // this thread's column of dY and dE (kDiv)
        if constexpr (kDiv) {
#pragma unroll
          for (int t = 0; t < kTB; ++t) {
            yc[t] = Ys[t * ldv + tid % dv];
            dc[t] = Vs[t * ldv + tid % dv];
          }
        }
#pragma unroll
        for (int u = 0; u < kRegs; ++u) {
          const int r = row_of(u, dv), j = col_of(u, dv);
          if (r < dk) {
            float rr = Acc[r * ldw + j];
#pragma unroll
            for (int t = 0; t < kTB; ++t)
              rr = fmaf(Qs[t * ldk + r], kDiv ? yc[t] : Ys[t * ldv + j], rr);
            Acc[r * ldw + j] = rr;
            if (mse) {
#pragma unroll
              for (int t = 0; t < kTB; ++t)
                kde[u] = fmaf(Ks[t * ldk + r], kDiv ? dc[t] : Vs[t * ldv + j], kde[u]);
            }
          }
        }
      }
    }
    // chunk start: dL/dW_s = R + sum_t k_t^T de_t is the previous chunk's G
    // (each thread updates the elements it accumulated)
#pragma unroll
    for (int u = 0; u < kRegs; ++u) {
      const int r = row_of(u, dv), j = col_of(u, dv);
      if (r < dk) {
        Acc[r * ldw + j] += kde[u];
        kde[u] = 0.f;
      }
    }
  }
  __syncthreads();
  float* dW = a.dW + (int64_t)bh * n;
  for (int x = tid; x < n; x += kNT) dW[x] = Acc[(x / dv) * ldw + x % dv];
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

bool ttt_linear_bwd_supported(int dk, int dv) {
  return dk >= 1 && dv >= 1 && dk <= kMaxD && dv <= kMaxD;
}

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
  const size_t smem = sizeof(float) * bwd_smem_floats(a.dk, a.dv);
  auto go = [&](auto kern, int nt) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) kern<<<(int)Z, nt, smem, s>>>(a);
    return e;
  };
  const bool small = a.dk <= 64 && a.dv <= 64;
  const int nt = threads_for(small ? 64 : 128);
  const bool div = nt % a.dk == 0 && nt % a.dv == 0;
  cudaError_t e;
  if (bf16) {
    if (small)
      e = div ? go(ttt_linear_bwd_kernel<__nv_bfloat16, true, 64>, nt)
              : go(ttt_linear_bwd_kernel<__nv_bfloat16, false, 64>, nt);
    else
      e = div ? go(ttt_linear_bwd_kernel<__nv_bfloat16, true, 128>, nt)
              : go(ttt_linear_bwd_kernel<__nv_bfloat16, false, 128>, nt);
  } else {
    if (small)
      e = div ? go(ttt_linear_bwd_kernel<float, true, 64>, nt)
              : go(ttt_linear_bwd_kernel<float, false, 64>, nt);
    else
      e = div ? go(ttt_linear_bwd_kernel<float, true, 128>, nt)
              : go(ttt_linear_bwd_kernel<float, false, 128>, nt);
  }
  if (e != cudaSuccess) return e;
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
