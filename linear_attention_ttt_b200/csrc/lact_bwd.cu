// LaCT SwiGLU layer backward (training): gradients of a scalar objective
// through the LaCT forward, given dL/dy and optionally dL/d(final weights).
//
// The forward ("Test-Time Training Done Right" review, sections 3.2-3.3 and
// 4 / Figure 3), per (batch, head) and chunk c with weights w = (W1, W2, W3)
// at the chunk start:
//   apply      Y_c = f_w(Q_c) (causal; after the update when causal = 0),
//              f(x) = W2 (silu(W1 x) * W3 x)
//   gradient   with H1 = K W1^T, H3 = K W3^T, Vt = diag(eta) V, Gz = -Vt W2,
//              Ak = silu(H1) H3, dH3 = Gz silu(H1), dH1 = Gz H3 silu'(H1):
//              G1 = dH1^T K, G3 = dH3^T K, G2 = -Vt^T Ak
//   Muon       G <- NS5(G): X0 = G / (||G||_F + eps), X <- X P(X^T X) with
//              P(M) = a I + b M + c M^2 (tall form; a wide G is transposed)
//   step       U = w - G, then every row of U rescaled to the norm rho the
//              row had in the initial weights (a zero row is kept).
// The backward walks the chunks in reverse. With dW the gradient of the
// weights after chunk c:
//   renorm     dU_r = (rho_r / |U_r|)(dW_r - (dW_r . u_r) u_r), u_r = U_r/|U_r|,
//              d rho_r += dW_r . u_r
//   Muon       per iteration, from dX': dP = X^T dX', dM = b dP + c (dP M + M dP),
//              dX = dX' P + X (dM + dM^T); then the normalisation
//   gradient   (second order) with the upstream dG1, dG2, dG3:
//              d(dH1) = K dG1^T, d(dH3) = K dG3^T, dAk = -Vt dG2,
//              dK += dH1 dG1 + dH3 dG3 + dH1' W1 + dH3' W3,
//              dVt = -Ak dG2^T - dGz W2^T, where
//              dGz = d(dH1) H3 silu' + d(dH3) silu,
//              dH3' = d(dH1) Gz silu' + dAk silu,
//              dH1' = d(dH1) Gz H3 silu'' + d(dH3) Gz silu' + dAk H3 silu',
//              dW1 += dH1'^T K, dW3 += dH3'^T K, dW2 += -Vt^T dGz,
//              dv = eta dVt, deta = sum over columns of dVt * V
//   apply      the SwiGLU backward of Y_c = f_w(Q_c)
// and finally the initial weights also receive d rho through rho = |W_r|.
// silu'(x) = s (1 + x (1 - s)) and silu''(x) = s (1 - s)(2 + x (1 - 2 s)),
// s = sigmoid(x).
//
// fp32 arithmetic throughout (batched fp32 GEMMs on the CUDA cores and
// elementwise / row kernels), orchestrated chunk by chunk from the host over
// all (batch, head) pairs at once. A forward pass in the same fp32 arithmetic
// stores the start weights of every chunk.
#include <cstring>
#include <vector>

#include "lact.cuh"

namespace ttt {
namespace {

// ---------------------------------------------------------------------------
// Batched fp32 GEMM: C[z] = alpha op(A[z]) op(B[z]) + beta C[z], op(A) M x K,
// op(B) K x N; tA: A stored K x M (A[k * lda + m]); tB: B stored N x K.
// 64 x 64 output tiles, 256 threads with 4 x 4 outputs each, K steps of 16,
// the next step's operands fetched into registers during the current one.
// With blockIdx.z = split * Z + z, split s covers one K range and writes its
// partial tile to slab (split * Z + z) of C (see Ctx::gemm).
// ---------------------------------------------------------------------------
constexpr int kGT = 64, kGK = 16;

struct GemmArgs {
  const float* A;
  const float* B;
  float* C;
  int M, N, K, lda, ldb, ldc, tA, tB;
  int64_t sA, sB, sC;
  float alpha, beta;
  int Z, kper;  // blockIdx.z = split * Z + z; split s covers K range [s kper, (s + 1) kper)
};

__global__ void __launch_bounds__(256) bgemm_kernel(GemmArgs g) {
  __shared__ float As[kGK][kGT + 4];
  __shared__ float Bs[kGK][kGT + 4];
  const int zz = blockIdx.z, z = zz % g.Z, sp = zz / g.Z;
  const float* A = g.A + z * g.sA;
  const float* B = g.B + z * g.sB;
  float* C = g.C + zz * g.sC;  // split partials (sp > 0) go to consecutive slabs
  const int kb = sp * g.kper, ke = min(g.K, kb + g.kper);
  const int m0 = blockIdx.y * kGT, n0 = blockIdx.x * kGT;
  const int tid = threadIdx.x, tm = tid / 16, tn = tid % 16;
  float acc[4][4] = {};
  // The next K step's operands are fetched into registers while the current
  // step is computed (every load of a step is issued before its stores).
  constexpr int kPer = kGK * kGT / 256;  // operand elements per thread and step
  float ra[kPer], rb[kPer];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + 256 * i;
      int kk, mm;
      if (g.tA) { mm = e % kGT; kk = e / kGT; } else { kk = e % kGK; mm = e / kGK; }
      const int gm = m0 + mm, gk = k0 + kk;
      ra[i] = (gm < g.M && gk < ke)
                  ? (g.tA ? A[(int64_t)gk * g.lda + gm] : A[(int64_t)gm * g.lda + gk])
                  : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + 256 * i;
      int kk, nn;
      if (g.tB) { kk = e % kGK; nn = e / kGK; } else { nn = e % kGT; kk = e / kGT; }
      const int gn = n0 + nn, gk = k0 + kk;
      rb[i] = (gn < g.N && gk < ke)
                  ? (g.tB ? B[(int64_t)gn * g.ldb + gk] : B[(int64_t)gk * g.ldb + gn])
                  : 0.f;
    }
  };
  auto stage = [&]() {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = tid + 256 * i;
      if (g.tA) As[e / kGT][e % kGT] = ra[i]; else As[e % kGK][e / kGK] = ra[i];
      if (g.tB) Bs[e % kGK][e / kGK] = rb[i]; else Bs[e / kGT][e % kGT] = rb[i];
    }
  };
  if (kb < ke) fetch(kb);
  for (int k0 = kb; k0 < ke; k0 += kGK) {
    stage();
    __syncthreads();
    if (k0 + kGK < ke) fetch(k0 + kGK);
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][tm + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tn + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + tm + 16 * i, n = n0 + tn + 16 * j;
      if (m < g.M && n < g.N) {
        float* c = C + (int64_t)m * g.ldc + n;
        *c = g.alpha * acc[i][j] + (g.beta != 0.f ? g.beta * *c : 0.f);
      }
    }
}

// C[z] = alpha sum_s part[s][z] + beta C[z], the split-K partials summed in
// split order (deterministic).
__global__ void splitk_reduce_kernel(const float* part, float* C, int Z, int M, int N, int ldc,
                                     int64_t sC, int splits, float alpha, float beta) {
  const int64_t mn = (int64_t)M * N, n = (int64_t)Z * mn;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int z = (int)(i / mn);
    const int64_t r = i % mn;
    const int m = (int)(r / N), c = (int)(r % N);
    float acc = 0.f;
    for (int sp = 0; sp < splits; ++sp) acc += part[((int64_t)sp * Z + z) * mn + r];
    float* o = C + z * sC + (int64_t)m * ldc + c;
    *o = alpha * acc + (beta != 0.f ? beta * *o : 0.f);
  }
}

// ---------------------------------------------------------------------------
// Elementwise and row kernels over [Z][rows][cols] buffers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + expf(-x)); }

enum EwOp : int {
  EW_KEY = 0,      // in: H1, H3, Gz       out: Ak, dH1f, dH3f
  EW_KEY_BWD = 1,  // in: H1, H3, Gz, d(dH1) in o0, d(dH3) in o1, dAk in o2
                   // out (in place): o0 = dGz, o1 = dH1', o2 = dH3'
  EW_APPLY = 2,    // in: Hq1, Hq3        out: Aq
  EW_APPLY_BWD = 3,  // in: Hq1, Hq3, dAq  out: dHq1, dHq3
  EW_SUB = 4,      // o0 = i0 - i1
  EW_POLY = 5,     // o0 = a I + b i0 + c i1  (square matrices of side `cols`)
  EW_SYM = 6,      // o0 = i0 + i0^T (square, per z)
  EW_TRANS = 7,    // o0[z][c][r] = i0[z][r][c]
  EW_AXPBY = 8,    // o0 = a i0 + b i1
};

struct EwArgs {
  const float* in[3];
  float* out[3];
  int64_t n;         // elements per z
  int Z, rows, cols;
  float a, b, c;
  int op;
};

__global__ void ew_kernel(EwArgs e) {
  const int64_t total = e.n * e.Z;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    switch (e.op) {
      case EW_KEY: {
        const float h1 = e.in[0][i], h3 = e.in[1][i], gz = e.in[2][i];
        const float s = sigm(h1), sl = h1 * s, sp = s * (1.f + h1 * (1.f - s));
        e.out[0][i] = sl * h3;
        e.out[1][i] = gz * h3 * sp;
        e.out[2][i] = gz * sl;
        break;
      }
      case EW_KEY_BWD: {
        const float h1 = e.in[0][i], h3 = e.in[1][i], gz = e.in[2][i];
        const float d1 = e.out[0][i], d3 = e.out[1][i], dak = e.out[2][i];
        const float s = sigm(h1), sl = h1 * s, sp = s * (1.f + h1 * (1.f - s));
        const float spp = s * (1.f - s) * (2.f + h1 * (1.f - 2.f * s));
        e.out[0][i] = d1 * h3 * sp + d3 * sl;                        // dGz
        e.out[1][i] = d1 * gz * h3 * spp + d3 * gz * sp + dak * h3 * sp;  // dH1'
        e.out[2][i] = d1 * gz * sp + dak * sl;                       // dH3'
        break;
      }
      case EW_APPLY: {
        const float h1 = e.in[0][i], h3 = e.in[1][i];
        e.out[0][i] = h1 * sigm(h1) * h3;
        break;
      }
      case EW_APPLY_BWD: {
        const float h1 = e.in[0][i], h3 = e.in[1][i], da = e.in[2][i];
        const float s = sigm(h1), sp = s * (1.f + h1 * (1.f - s));
        e.out[0][i] = da * h3 * sp;
        e.out[1][i] = da * h1 * s;
        break;
      }
      case EW_SUB:
        e.out[0][i] = e.in[0][i] - e.in[1][i];
        break;
      case EW_POLY: {
        const int64_t w = i % e.n;
        const int r = (int)(w / e.cols), c = (int)(w % e.cols);
        e.out[0][i] = (r == c ? e.a : 0.f) + e.b * e.in[0][i] + e.c * e.in[1][i];
        break;
      }
      case EW_SYM: {
        const int64_t z = i / e.n, w = i % e.n;
        const int r = (int)(w / e.cols), c = (int)(w % e.cols);
        e.out[0][i] = e.in[0][i] + e.in[0][z * e.n + (int64_t)c * e.cols + r];
        break;
      }
      case EW_TRANS: {
        const int64_t z = i / e.n, w = i % e.n;
        const int r = (int)(w / e.cols), c = (int)(w % e.cols);
        e.out[0][z * e.n + (int64_t)c * e.rows + r] = e.in[0][i];
        break;
      }
      case EW_AXPBY:
        e.out[0][i] = e.a * e.in[0][i] + e.b * e.in[1][i];
        break;
    }
  }
}

// Per (z, row): squared norm of U's row (mode 0, into nrm), or the renorm
// step (mode 1): W = rho U / |U| (zero rows kept), or its backward (mode 2):
// dU = (rho/|U|)(dW - (dW.u) u), drho += dW.u, for rows of `cols` values.
// One warp per row.
struct RowOpArgs {
  const float* U;
  float* W;          // mode 1 output
  const float* dW;   // mode 2
  float* dU;         // mode 2 output
  float* rho;        // [Z][rows]: mode 0 output, modes 1-2 input
  float* drho;       // mode 2 accumulation
  int Z, rows, cols, mode;
};

__global__ void rowop_kernel(RowOpArgs a) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= a.Z * a.rows) return;
  const float* u = a.U + (int64_t)gw * a.cols;
  float ss = 0.f;
  for (int c = lane; c < a.cols; c += 32) ss = fmaf(u[c], u[c], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float nrm = sqrtf(ss);
  if (a.mode == 0) {
    if (lane == 0) a.rho[gw] = nrm;
    return;
  }
  const float rho = a.rho[gw];
  if (a.mode == 1) {
    const float s = nrm > 0.f ? rho / nrm : 1.f;
    for (int c = lane; c < a.cols; c += 32) a.W[(int64_t)gw * a.cols + c] = u[c] * s;
    return;
  }
  const float* dw = a.dW + (int64_t)gw * a.cols;
  float* du = a.dU + (int64_t)gw * a.cols;
  if (!(nrm > 0.f)) {
    for (int c = lane; c < a.cols; c += 32) du[c] = dw[c];
    return;
  }
  const float inv = 1.f / nrm;
  float pr = 0.f;
  for (int c = lane; c < a.cols; c += 32) pr = fmaf(dw[c], u[c] * inv, pr);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) pr += __shfl_xor_sync(0xffffffffu, pr, o);
  if (lane == 0) a.drho[gw] += pr;
  for (int c = lane; c < a.cols; c += 32) du[c] = rho * inv * (dw[c] - pr * u[c] * inv);
}

// Per z: s[z] = sum of x[z] * y[z] over n elements (one block per z).
__global__ void dot_kernel(const float* x, const float* y, float* s, int64_t n) {
  __shared__ float red[32];
  const int z = blockIdx.x;
  float acc = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) acc = fmaf(x[z * n + i], y[z * n + i], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    s[z] = t;
  }
}

// NS normalisation: mode 0: X0 = X / (sqrt(s) + eps); mode 1 (backward):
// dG = dX / (r + eps) - X (X . dX) / ((r + eps)^2 r), r = sqrt(s), t = X . dX.
__global__ void ns_norm_kernel(const float* X, const float* dX, float* out, const float* s,
                               const float* t, int64_t n, int Z, float eps, int mode) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n * Z;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int z = (int)(i / n);
    const float r = sqrtf(s[z]), d = r + eps;
    if (mode == 0) out[i] = X[i] / d;
    else out[i] = r > 0.f ? dX[i] / d - X[i] * t[z] / (d * d * r) : dX[i] / d;
  }
}

// Token tensors <-> contiguous fp32 chunk buffers [Z][bc][d].
template <typename T>
__global__ void gather_kernel(float* dst, TokView src, int H, int t0, int bc, int d, int Z) {
  const int64_t total = (int64_t)Z * bc * d;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % d);
    const int t = (int)((i / d) % bc);
    const int z = (int)(i / ((int64_t)d * bc));
    const int b = z / H, h = z % H;
    dst[i] = to_f32(static_cast<const T*>(src.p)[b * src.sb + h * src.sh + (int64_t)(t0 + t) * src.st + c]);
  }
}
template <typename T>
__global__ void scatter_kernel(TokViewMut dst, const float* src, int H, int t0, int bc, int d,
                               int Z) {
  const int64_t total = (int64_t)Z * bc * d;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % d);
    const int t = (int)((i / d) % bc);
    const int z = (int)(i / ((int64_t)d * bc));
    const int b = z / H, h = z % H;
    static_cast<T*>(dst.p)[b * dst.sb + h * dst.sh + (int64_t)(t0 + t) * dst.st + c] = T(src[i]);
  }
}
// eta of the chunk [Z][bc]; Vt = eta V; and the backward's dv = eta dVt,
// deta = sum_c dVt V (mode 1)
__global__ void eta_kernel(const float* V, const float* dVt, float* Vt_or_dv, float* etac,
                           float* deta_out, EtaView eta, int H, int t0, int bc, int d, int Z,
                           int mode) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= Z * bc) return;
  const int z = row / bc, t = row % bc, b = z / H, h = z % H;
  const float e = eta.p[b * eta.sb + h * eta.sh + (int64_t)(t0 + t) * eta.st];
  if (mode == 0) {
    if (lane == 0) etac[row] = e;
    for (int c = lane; c < d; c += 32) Vt_or_dv[(int64_t)row * d + c] = e * V[(int64_t)row * d + c];
    return;
  }
  float acc = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float g = dVt[(int64_t)row * d + c];
    acc = fmaf(g, V[(int64_t)row * d + c], acc);
    Vt_or_dv[(int64_t)row * d + c] = e * g;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) deta_out[row] = acc;
}
// deta [B,H,T] (contiguous) <- per-chunk values
__global__ void deta_scatter_kernel(float* deta, const float* src, int T, int t0, int bc, int Z) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < Z * bc; i += gridDim.x * blockDim.x) {
    const int z = i / bc, t = i % bc;
    deta[(int64_t)z * T + t0 + t] = src[i];
  }
}
// dW_init += (drho / rho) W_init per row (rho > 0); one warp per row
__global__ void rho_grad_kernel(float* dW, const float* W, const float* rho, const float* drho,
                                int Z, int rows, int cols) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= Z * rows) return;
  const float r = rho[gw];
  if (!(r > 0.f)) return;
  const float s = drho[gw] / r;
  for (int c = lane; c < cols; c += 32) dW[(int64_t)gw * cols + c] += s * W[(int64_t)gw * cols + c];
}
// per-head weights [H][n] (shared over the batch) -> [Z][n] copies, or the
// batch sum of [Z][n] into [H][n] (mode 1)
__global__ void bcast_kernel(float* dst, const float* src, int64_t n, int B, int H, int mode) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)H * n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int h = (int)(i / n);
    const int64_t w = i % n;
    if (mode == 0) {
      for (int b = 0; b < B; ++b) dst[((int64_t)b * H + h) * n + w] = src[i];
    } else {
      float s = 0.f;
      for (int b = 0; b < B; ++b) s += src[((int64_t)b * H + h) * n + w];
      dst[i] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct Ctx {
  cudaStream_t s;
  bool ok = true;
  void check(cudaError_t e) {
    if (e != cudaSuccess) ok = false;
  }
  int grid(int64_t n, int per = 256) {
    const int64_t b = (n + per - 1) / per;
    return (int)(b < 4096 ? (b < 1 ? 1 : b) : 4096);
  }
  // split-K scratch: room for kMaxSplit partial [M][N] slabs per z
  float* sk = nullptr;
  int64_t sk_mn = 0;
  static constexpr int kMaxSplit = 8;
  // C = alpha op(A) op(B) + beta C for all z. A product with few output tiles
  // and a long K (the token reductions of the weight gradients) is split over
  // K into partial slabs, summed by splitk_reduce_kernel in split order.
  void gemm(int Z, int M, int N, int K, const float* A, int lda, int64_t sA, bool tA,
            const float* B, int ldb, int64_t sB, bool tB, float* C, int ldc, int64_t sC,
            float alpha = 1.f, float beta = 0.f) {
    if (M == 0 || N == 0 || Z == 0) return;
    const int tiles = Z * ((N + kGT - 1) / kGT) * ((M + kGT - 1) / kGT);
    int splits = 1;
    if (sk && (int64_t)M * N <= sk_mn && tiles < 148 && K >= 8 * kGK) {
      splits = (2 * 148 + tiles - 1) / tiles;
      const int by_k = K / (4 * kGK);  // at least four K steps per split
      if (splits > by_k) splits = by_k;
      if (splits > kMaxSplit) splits = kMaxSplit;
    }
    if (splits <= 1) {
      GemmArgs g{A, B, C, M, N, K, lda, ldb, ldc, tA, tB, sA, sB, sC, alpha, beta, Z, K};
      dim3 grid((N + kGT - 1) / kGT, (M + kGT - 1) / kGT, Z);
      bgemm_kernel<<<grid, 256, 0, s>>>(g);
      check(cudaGetLastError());
      return;
    }
    const int ksteps = (K + kGK - 1) / kGK;
    const int kper = (ksteps + splits - 1) / splits * kGK;
    splits = (K + kper - 1) / kper;
    GemmArgs g{A, B, sk, M, N, K, lda, ldb, N, tA, tB, sA, sB, (int64_t)M * N, 1.f, 0.f, Z, kper};
    dim3 grid((N + kGT - 1) / kGT, (M + kGT - 1) / kGT, Z * splits);
    bgemm_kernel<<<grid, 256, 0, s>>>(g);
    check(cudaGetLastError());
    splitk_reduce_kernel<<<grid1((int64_t)Z * M * N), 256, 0, s>>>(sk, C, Z, M, N, ldc, sC, splits,
                                                                   alpha, beta);
    check(cudaGetLastError());
  }
  int grid1(int64_t n) { return grid(n); }
  void ew(int op, int Z, int64_t n, std::initializer_list<const float*> in,
          std::initializer_list<float*> out, int rows = 0, int cols = 0, float a = 0.f,
          float b = 0.f, float c = 0.f) {
    EwArgs e;
    memset(&e, 0, sizeof(e));
    int i = 0;
    for (const float* p : in) e.in[i++] = p;
    i = 0;
    for (float* p : out) e.out[i++] = p;
    e.n = n;
    e.Z = Z;
    e.rows = rows;
    e.cols = cols;
    e.a = a;
    e.b = b;
    e.c = c;
    e.op = op;
    ew_kernel<<<grid(n * Z), 256, 0, s>>>(e);
    check(cudaGetLastError());
  }
  void rowop(int mode, int Z, int rows, int cols, const float* U, float* W, const float* dW,
             float* dU, float* rho, float* drho) {
    RowOpArgs r{U, W, dW, dU, rho, drho, Z, rows, cols, mode};
    const int warps = Z * rows;
    rowop_kernel<<<(warps * 32 + 255) / 256, 256, 0, s>>>(r);
    check(cudaGetLastError());
  }
};

}  // namespace

bool lact_bwd_supported(const LactArgs& a) {
  return a.dk <= 256 && a.dv <= 256 && a.dh <= 1024 && a.B * a.H <= 65535 &&
         (a.update_rule == LACT_UPDATE_GD || a.update_rule == LACT_UPDATE_MUON);
}

ttt_status lact_backward(const LactArgs& a, const LactBwdArgs& g, cudaStream_t st) {
  if (!lact_bwd_supported(a)) return TTT_ERR_UNSUPPORTED;
  Ctx x;
  x.s = st;
  const int Z = a.B * a.H, dk = a.dk, dv = a.dv, dh = a.dh, T = a.T;
  const int chunk = T > 0 ? (a.chunk < T ? a.chunk : T) : 1;
  const int nch = T > 0 ? (T + chunk - 1) / chunk : 0;
  const bool muon = a.update_rule == LACT_UPDATE_MUON;
  const int64_t nW[3] = {(int64_t)dh * dk, (int64_t)dv * dh, (int64_t)dh * dk};
  const int rowsW[3] = {dh, dv, dh}, colsW[3] = {dk, dh, dk};
  const int64_t nWall = nW[0] + nW[1] + nW[2];
  // tall form of each gradient for Newton-Schulz: m x n with m >= n
  int tm[3], tn[3];
  for (int m = 0; m < 3; ++m) {
    tm[m] = rowsW[m] >= colsW[m] ? rowsW[m] : colsW[m];
    tn[m] = rowsW[m] >= colsW[m] ? colsW[m] : rowsW[m];
  }
  const int nmax = tn[0] > tn[1] ? tn[0] : tn[1];  // Newton-Schulz small side
  const int64_t bd = (int64_t)chunk * (dk > dv ? dk : dv), bh = (int64_t)chunk * dh;
  const int64_t nn_max = (int64_t)nmax * nmax;
  const int64_t mn_max = nW[0] > nW[1] ? nW[0] : nW[1];

  // workspace layout (floats, per z unless noted)
  size_t off = 0;
  auto take = [&](int64_t per_z) {
    const size_t o = off;
    off += (size_t)Z * per_z;
    off = (off + 63) / 64 * 64;
    return o;
  };
  const size_t o_ck = take((int64_t)(nch > 0 ? nch : 1) * nWall);
  size_t o_w0[3], o_rho[3], o_drho[3], o_dW[3], o_dn[3], o_G[3], o_U[3];
  for (int m = 0; m < 3; ++m) {
    o_w0[m] = take(nW[m]);
    o_rho[m] = take(rowsW[m]);
    o_drho[m] = take(rowsW[m]);
    o_dW[m] = take(nW[m]);
    o_dn[m] = take(nW[m]);
    o_G[m] = take(nW[m]);
    o_U[m] = take(nW[m]);
  }
  const size_t o_Qc = take(bd), o_Kc = take(bd), o_Vc = take(bd), o_Vt = take(bd), o_dY = take(bd),
               o_dK = take(bd), o_dVt = take(bd), o_dQ = take(bd), o_eta = take(chunk),
               o_deta = take(chunk);
  const size_t o_H1 = take(bh), o_H3 = take(bh), o_Gz = take(bh), o_Ak = take(bh), o_D1 = take(bh),
               o_D3 = take(bh), o_E0 = take(bh), o_E1 = take(bh), o_E2 = take(bh);
  // Newton-Schulz caches of one matrix: X_0..X_5 (m x n), M_0..4, P_0..4 (n x n)
  size_t o_X[6], o_M[5], o_P[5];
  for (int i = 0; i < 6; ++i) o_X[i] = take(mn_max);
  for (int i = 0; i < 5; ++i) {
    o_M[i] = take(nn_max);
    o_P[i] = take(nn_max);
  }
  const size_t o_Xt = take(mn_max), o_dX = take(mn_max), o_dX2 = take(mn_max), o_dP = take(nn_max),
               o_dM = take(nn_max), o_tmp = take(nn_max), o_red = take(2);
  // split-K slabs for the weight-shaped products; only small batches have
  // fewer output tiles than SMs, so larger ones get no scratch and no split
  const int64_t sk_mn = Z <= 16 ? mn_max : 0;
  const size_t o_sk = take(Ctx::kMaxSplit * sk_mn);
  const size_t bytes = off * sizeof(float);
  void* base = nullptr;
  if (scratch_alloc(&base, bytes, st) != cudaSuccess) return TTT_ERR_ALLOC;
  float* F = static_cast<float*>(base);
  auto P = [&](size_t o) { return F + o; };
  x.sk = sk_mn > 0 ? P(o_sk) : nullptr;
  x.sk_mn = sk_mn;

  const float* Win[3] = {a.W1, a.W2, a.W3};
  // initial weights per z, row norms
  for (int m = 0; m < 3; ++m) {
    if (a.w_sb[m]) {
      x.check(cudaMemcpyAsync(P(o_w0[m]), Win[m], sizeof(float) * Z * nW[m],
                              cudaMemcpyDeviceToDevice, st));
    } else {
      bcast_kernel<<<x.grid((int64_t)a.H * nW[m]), 256, 0, st>>>(P(o_w0[m]), Win[m], nW[m], a.B,
                                                                a.H, 0);
      x.check(cudaGetLastError());
    }
    x.rowop(0, Z, rowsW[m], colsW[m], P(o_w0[m]), nullptr, nullptr, nullptr, P(o_rho[m]),
            nullptr);
    x.check(cudaMemsetAsync(P(o_drho[m]), 0, sizeof(float) * Z * rowsW[m], st));
  }
  auto ck = [&](int c, int m) {
    int64_t o = (int64_t)c * nWall + (m > 0 ? nW[0] : 0) + (m > 1 ? nW[1] : 0);
    return P(o_ck) + o * Z;  // [c][m] block of Z matrices
  };

  auto gather = [&](float* dst, const TokView& v, int t0, int bc, int d) {
    if (a.dtype == TTT_BF16)
      gather_kernel<__nv_bfloat16><<<x.grid((int64_t)Z * bc * d), 256, 0, st>>>(dst, v, a.H, t0, bc, d, Z);
    else
      gather_kernel<float><<<x.grid((int64_t)Z * bc * d), 256, 0, st>>>(dst, v, a.H, t0, bc, d, Z);
    x.check(cudaGetLastError());
  };
  auto scatter = [&](const TokViewMut& v, const float* src, int t0, int bc, int d) {
    if (a.dtype == TTT_BF16)
      scatter_kernel<__nv_bfloat16><<<x.grid((int64_t)Z * bc * d), 256, 0, st>>>(v, src, a.H, t0, bc, d, Z);
    else
      scatter_kernel<float><<<x.grid((int64_t)Z * bc * d), 256, 0, st>>>(v, src, a.H, t0, bc, d, Z);
    x.check(cudaGetLastError());
  };

  // Newton-Schulz of G[m] (in place, result in G[m]); caches X_k, M_k, P_k
  auto ns_forward = [&](int m) {
    const int M_ = tm[m], N_ = tn[m];
    const int64_t mn = (int64_t)M_ * N_, nn = (int64_t)N_ * N_;
    const bool wide = rowsW[m] < colsW[m];
    float* Xsrc = P(o_G[m]);
    if (wide) {
      x.ew(EW_TRANS, Z, nW[m], {P(o_G[m])}, {P(o_Xt)}, rowsW[m], colsW[m]);
      Xsrc = P(o_Xt);
    } else {
      x.check(cudaMemcpyAsync(P(o_Xt), P(o_G[m]), sizeof(float) * Z * mn, cudaMemcpyDeviceToDevice, st));
      Xsrc = P(o_Xt);
    }
    dot_kernel<<<Z, 256, 0, st>>>(Xsrc, Xsrc, P(o_red), mn);
    x.check(cudaGetLastError());
    ns_norm_kernel<<<x.grid(Z * mn), 256, 0, st>>>(Xsrc, nullptr, P(o_X[0]), P(o_red), nullptr, mn,
                                                   Z, 1e-7f, 0);
    x.check(cudaGetLastError());
    for (int k = 0; k < 5; ++k) {
      x.gemm(Z, N_, N_, M_, P(o_X[k]), N_, mn, true, P(o_X[k]), N_, mn, false, P(o_M[k]), N_, nn);
      x.gemm(Z, N_, N_, N_, P(o_M[k]), N_, nn, false, P(o_M[k]), N_, nn, false, P(o_tmp), N_, nn);
      x.ew(EW_POLY, Z, nn, {P(o_M[k]), P(o_tmp)}, {P(o_P[k])}, N_, N_, 3.4445f, -4.7750f, 2.0315f);
      x.gemm(Z, M_, N_, N_, P(o_X[k]), N_, mn, false, P(o_P[k]), N_, nn, false, P(o_X[k + 1]), N_, mn);
    }
    if (wide)
      x.ew(EW_TRANS, Z, mn, {P(o_X[5])}, {P(o_G[m])}, M_, N_);
    else
      x.check(cudaMemcpyAsync(P(o_G[m]), P(o_X[5]), sizeof(float) * Z * mn, cudaMemcpyDeviceToDevice, st));
  };
  // backward of ns_forward(m): dOut in `dG` (rows x cols layout), result in place
  auto ns_backward = [&](int m, float* dG) {
    const int M_ = tm[m], N_ = tn[m];
    const int64_t mn = (int64_t)M_ * N_, nn = (int64_t)N_ * N_;
    const bool wide = rowsW[m] < colsW[m];
    if (wide)
      x.ew(EW_TRANS, Z, nW[m], {dG}, {P(o_dX)}, rowsW[m], colsW[m]);
    else
      x.check(cudaMemcpyAsync(P(o_dX), dG, sizeof(float) * Z * mn, cudaMemcpyDeviceToDevice, st));
    for (int k = 4; k >= 0; --k) {
      // dP = X_k^T dX; dM = b dP + c (dP M + M dP)
      x.gemm(Z, N_, N_, M_, P(o_X[k]), N_, mn, true, P(o_dX), N_, mn, false, P(o_dP), N_, nn);
      x.gemm(Z, N_, N_, N_, P(o_dP), N_, nn, false, P(o_M[k]), N_, nn, false, P(o_dM), N_, nn, 2.0315f);
      x.gemm(Z, N_, N_, N_, P(o_M[k]), N_, nn, false, P(o_dP), N_, nn, false, P(o_dM), N_, nn, 2.0315f,
             1.f);
      x.ew(EW_AXPBY, Z, nn, {P(o_dP), P(o_dM)}, {P(o_dM)}, 0, 0, -4.7750f, 1.f);
      x.ew(EW_SYM, Z, nn, {P(o_dM)}, {P(o_tmp)}, N_, N_);
      // dX <- dX P + X_k (dM + dM^T)
      x.gemm(Z, M_, N_, N_, P(o_dX), N_, mn, false, P(o_P[k]), N_, nn, false, P(o_dX2), N_, mn);
      x.gemm(Z, M_, N_, N_, P(o_X[k]), N_, mn, false, P(o_tmp), N_, nn, false, P(o_dX2), N_, mn, 1.f,
             1.f);
      x.check(cudaMemcpyAsync(P(o_dX), P(o_dX2), sizeof(float) * Z * mn, cudaMemcpyDeviceToDevice, st));
    }
    // normalisation: X = tall G (o_Xt holds it from the forward of this chunk)
    dot_kernel<<<Z, 256, 0, st>>>(P(o_Xt), P(o_Xt), P(o_red), mn);
    dot_kernel<<<Z, 256, 0, st>>>(P(o_Xt), P(o_dX), P(o_red) + Z, mn);
    x.check(cudaGetLastError());
    ns_norm_kernel<<<x.grid(Z * mn), 256, 0, st>>>(P(o_Xt), P(o_dX), P(o_dX2), P(o_red),
                                                   P(o_red) + Z, mn, Z, 1e-7f, 1);
    x.check(cudaGetLastError());
    if (wide)
      x.ew(EW_TRANS, Z, mn, {P(o_dX2)}, {dG}, M_, N_);
    else
      x.check(cudaMemcpyAsync(dG, P(o_dX2), sizeof(float) * Z * mn, cudaMemcpyDeviceToDevice, st));
  };
  // Every per-chunk buffer holds the chunk's bc tokens per z contiguously
  // (z stride bc x d), so the GEMM strides follow bc. Key-side forward of a
  // chunk at weights w: H1, H3, Gz, Ak, dH1f, dH3f and the gradients G.
  auto run_key_forward = [&](float* const (&w)[3], int bc) {
    const int64_t sbk = (int64_t)bc * dk, sbv = (int64_t)bc * dv, sbh = (int64_t)bc * dh;
    x.gemm(Z, bc, dh, dk, P(o_Kc), dk, sbk, false, w[0], dk, nW[0], true, P(o_H1), dh, sbh);
    x.gemm(Z, bc, dh, dk, P(o_Kc), dk, sbk, false, w[2], dk, nW[2], true, P(o_H3), dh, sbh);
    x.gemm(Z, bc, dh, dv, P(o_Vt), dv, sbv, false, w[1], dh, nW[1], false, P(o_Gz), dh, sbh, -1.f);
    x.ew(EW_KEY, Z, sbh, {P(o_H1), P(o_H3), P(o_Gz)}, {P(o_Ak), P(o_D1), P(o_D3)});
    x.gemm(Z, dh, dk, bc, P(o_D1), dh, sbh, true, P(o_Kc), dk, sbk, false, P(o_G[0]), dk, nW[0]);
    x.gemm(Z, dh, dk, bc, P(o_D3), dh, sbh, true, P(o_Kc), dk, sbk, false, P(o_G[2]), dk, nW[2]);
    x.gemm(Z, dv, dh, bc, P(o_Vt), dv, sbv, true, P(o_Ak), dh, sbh, false, P(o_G[1]), dh, nW[1], -1.f);
  };

  // ---- forward in fp32: chunk-start weights ----
  float* wrun[3] = {P(o_dn[0]), P(o_dn[1]), P(o_dn[2])};  // running weights (dn reused)
  for (int m = 0; m < 3; ++m)
    x.check(cudaMemcpyAsync(wrun[m], P(o_w0[m]), sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
  for (int c = 0; c < nch && x.ok; ++c) {
    const int t0 = c * chunk, bc = (T - t0) < chunk ? (T - t0) : chunk;
    for (int m = 0; m < 3; ++m)
      x.check(cudaMemcpyAsync(ck(c, m), wrun[m], sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
    gather(P(o_Kc), a.k, t0, bc, dk);
    gather(P(o_Vc), a.v, t0, bc, dv);
    eta_kernel<<<(Z * bc * 32 + 255) / 256, 256, 0, st>>>(P(o_Vc), nullptr, P(o_Vt), P(o_eta),
                                                          nullptr, a.eta, a.H, t0, bc, dv, Z, 0);
    x.check(cudaGetLastError());
    run_key_forward(wrun, bc);
    if (muon)
      for (int m = 0; m < 3; ++m) ns_forward(m);
    for (int m = 0; m < 3; ++m) {
      x.ew(EW_SUB, Z, nW[m], {wrun[m], P(o_G[m])}, {P(o_U[m])});
      x.rowop(1, Z, rowsW[m], colsW[m], P(o_U[m]), wrun[m], nullptr, nullptr, P(o_rho[m]), nullptr);
    }
  }

  // ---- backward ----
  float* dW[3] = {P(o_dW[0]), P(o_dW[1]), P(o_dW[2])};
  float* dn[3] = {P(o_dn[0]), P(o_dn[1]), P(o_dn[2])};
  const float* dWf[3] = {g.dW1_final, g.dW2_final, g.dW3_final};
  for (int m = 0; m < 3; ++m) {
    if (dWf[m])
      x.check(cudaMemcpyAsync(dW[m], dWf[m], sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
    else
      x.check(cudaMemsetAsync(dW[m], 0, sizeof(float) * Z * nW[m], st));
  }
  // apply backward at weights w into dw (accumulating), for this chunk
  auto apply_backward = [&](float* const (&w)[3], float* const (&dw)[3], int t0, int bc) {
    const int64_t sbk = (int64_t)bc * dk, sbv = (int64_t)bc * dv, sbh = (int64_t)bc * dh;
    gather(P(o_Qc), a.q, t0, bc, dk);
    gather(P(o_dY), g.dy, t0, bc, dv);
    x.gemm(Z, bc, dh, dk, P(o_Qc), dk, sbk, false, w[0], dk, nW[0], true, P(o_E0), dh, sbh);  // Hq1
    x.gemm(Z, bc, dh, dk, P(o_Qc), dk, sbk, false, w[2], dk, nW[2], true, P(o_E1), dh, sbh);  // Hq3
    x.ew(EW_APPLY, Z, sbh, {P(o_E0), P(o_E1)}, {P(o_E2)});                                   // Aq
    x.gemm(Z, dv, dh, bc, P(o_dY), dv, sbv, true, P(o_E2), dh, sbh, false, dw[1], dh, nW[1], 1.f, 1.f);
    x.gemm(Z, bc, dh, dv, P(o_dY), dv, sbv, false, w[1], dh, nW[1], false, P(o_E2), dh, sbh);  // dAq
    x.ew(EW_APPLY_BWD, Z, sbh, {P(o_E0), P(o_E1), P(o_E2)}, {P(o_E0), P(o_E1)});  // dHq1, dHq3
    x.gemm(Z, bc, dk, dh, P(o_E0), dh, sbh, false, w[0], dk, nW[0], false, P(o_dQ), dk, sbk);
    x.gemm(Z, bc, dk, dh, P(o_E1), dh, sbh, false, w[2], dk, nW[2], false, P(o_dQ), dk, sbk, 1.f, 1.f);
    scatter(g.dq, P(o_dQ), t0, bc, dk);
    x.gemm(Z, dh, dk, bc, P(o_E0), dh, sbh, true, P(o_Qc), dk, sbk, false, dw[0], dk, nW[0], 1.f, 1.f);
    x.gemm(Z, dh, dk, bc, P(o_E1), dh, sbh, true, P(o_Qc), dk, sbk, false, dw[2], dk, nW[2], 1.f, 1.f);
  };
  for (int c = nch - 1; c >= 0 && x.ok; --c) {
    const int t0 = c * chunk, bc = (T - t0) < chunk ? (T - t0) : chunk;
    const int64_t sbk = (int64_t)bc * dk, sbv = (int64_t)bc * dv, sbh = (int64_t)bc * dh;
    float* w[3] = {ck(c, 0), ck(c, 1), ck(c, 2)};
    // non-causal: the chunk's outputs used the updated weights
    if (!a.causal) {
      float* wn[3] = {c + 1 < nch ? ck(c + 1, 0) : wrun[0], c + 1 < nch ? ck(c + 1, 1) : wrun[1],
                      c + 1 < nch ? ck(c + 1, 2) : wrun[2]};
      apply_backward(wn, dW, t0, bc);
    }
    gather(P(o_Kc), a.k, t0, bc, dk);
    gather(P(o_Vc), a.v, t0, bc, dv);
    eta_kernel<<<(Z * bc * 32 + 255) / 256, 256, 0, st>>>(P(o_Vc), nullptr, P(o_Vt), P(o_eta),
                                                          nullptr, a.eta, a.H, t0, bc, dv, Z, 0);
    x.check(cudaGetLastError());
    run_key_forward(w, bc);
    // renorm backward needs U = w - G~ for every matrix; G~ = NS(G) under Muon
    float* Gt[3] = {P(o_U[0]), P(o_U[1]), P(o_U[2])};
    for (int m = 0; m < 3; ++m) {
      if (muon) {
        x.check(cudaMemcpyAsync(P(o_dX2), P(o_G[m]), sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
        ns_forward(m);   // G[m] <- NS(G[m])
        x.ew(EW_SUB, Z, nW[m], {w[m], P(o_G[m])}, {Gt[m]});
        // restore the plain gradient (needed again for the Muon backward)
        x.check(cudaMemcpyAsync(P(o_G[m]), P(o_dX2), sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
      } else {
        x.ew(EW_SUB, Z, nW[m], {w[m], P(o_G[m])}, {Gt[m]});
      }
      // dn = dU (renorm backward), drho accumulated
      x.rowop(2, Z, rowsW[m], colsW[m], Gt[m], nullptr, dW[m], dn[m], P(o_rho[m]), P(o_drho[m]));
    }
    // dG~ = -dU; under Muon back through Newton-Schulz (caches recomputed per matrix)
    float* dG[3] = {P(o_U[0]), P(o_U[1]), P(o_U[2])};
    for (int m = 0; m < 3; ++m) {
      x.ew(EW_AXPBY, Z, nW[m], {dn[m], dn[m]}, {dG[m]}, 0, 0, -1.f, 0.f);
      if (muon) {
        x.check(cudaMemcpyAsync(P(o_dX2), P(o_G[m]), sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
        ns_forward(m);  // rebuild this matrix's caches (overwrites G[m])
        x.check(cudaMemcpyAsync(P(o_G[m]), P(o_dX2), sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
        ns_backward(m, dG[m]);
      }
    }
    // second order: through G(w, K, V, eta)
    x.gemm(Z, bc, dh, dk, P(o_Kc), dk, sbk, false, dG[0], dk, nW[0], true, P(o_E0), dh, sbh);  // d(dH1)
    x.gemm(Z, bc, dh, dk, P(o_Kc), dk, sbk, false, dG[2], dk, nW[2], true, P(o_E1), dh, sbh);  // d(dH3)
    x.gemm(Z, bc, dh, dv, P(o_Vt), dv, sbv, false, dG[1], dh, nW[1], false, P(o_E2), dh, sbh, -1.f);  // dAk
    x.gemm(Z, bc, dk, dh, P(o_D1), dh, sbh, false, dG[0], dk, nW[0], false, P(o_dK), dk, sbk);
    x.gemm(Z, bc, dk, dh, P(o_D3), dh, sbh, false, dG[2], dk, nW[2], false, P(o_dK), dk, sbk, 1.f, 1.f);
    x.gemm(Z, bc, dv, dh, P(o_Ak), dh, sbh, false, dG[1], dh, nW[1], true, P(o_dVt), dv, sbv, -1.f);
    x.ew(EW_KEY_BWD, Z, sbh, {P(o_H1), P(o_H3), P(o_Gz)}, {P(o_E0), P(o_E1), P(o_E2)});  // dGz, dH1', dH3'
    x.gemm(Z, bc, dv, dh, P(o_E0), dh, sbh, false, w[1], dh, nW[1], true, P(o_dVt), dv, sbv, -1.f, 1.f);
    x.gemm(Z, dv, dh, bc, P(o_Vt), dv, sbv, true, P(o_E0), dh, sbh, false, dn[1], dh, nW[1], -1.f, 1.f);
    x.gemm(Z, bc, dk, dh, P(o_E1), dh, sbh, false, w[0], dk, nW[0], false, P(o_dK), dk, sbk, 1.f, 1.f);
    x.gemm(Z, bc, dk, dh, P(o_E2), dh, sbh, false, w[2], dk, nW[2], false, P(o_dK), dk, sbk, 1.f, 1.f);
    x.gemm(Z, dh, dk, bc, P(o_E1), dh, sbh, true, P(o_Kc), dk, sbk, false, dn[0], dk, nW[0], 1.f, 1.f);
    x.gemm(Z, dh, dk, bc, P(o_E2), dh, sbh, true, P(o_Kc), dk, sbk, false, dn[2], dk, nW[2], 1.f, 1.f);
    scatter(g.dk, P(o_dK), t0, bc, dk);
    eta_kernel<<<(Z * bc * 32 + 255) / 256, 256, 0, st>>>(P(o_Vc), P(o_dVt), P(o_dY), P(o_eta),
                                                          P(o_deta), a.eta, a.H, t0, bc, dv, Z, 1);
    x.check(cudaGetLastError());
    scatter(g.dv, P(o_dY), t0, bc, dv);
    deta_scatter_kernel<<<x.grid((int64_t)Z * bc), 256, 0, st>>>(g.deta, P(o_deta), T, t0, bc, Z);
    x.check(cudaGetLastError());
    // causal: the chunk's outputs used the chunk-start weights
    if (a.causal) apply_backward(w, dn, t0, bc);
    for (int m = 0; m < 3; ++m) {
      float* t = dW[m];
      dW[m] = dn[m];
      dn[m] = t;
    }
  }
  // the initial weights also set the target norms rho
  for (int m = 0; m < 3; ++m) {
    const int warps = Z * rowsW[m];
    rho_grad_kernel<<<(warps * 32 + 255) / 256, 256, 0, st>>>(dW[m], P(o_w0[m]), P(o_rho[m]),
                                                              P(o_drho[m]), Z, rowsW[m], colsW[m]);
    x.check(cudaGetLastError());
  }
  float* outW[3] = {g.dW1, g.dW2, g.dW3};
  for (int m = 0; m < 3; ++m) {
    if (a.w_sb[m]) {
      x.check(cudaMemcpyAsync(outW[m], dW[m], sizeof(float) * Z * nW[m], cudaMemcpyDeviceToDevice, st));
    } else {
      bcast_kernel<<<x.grid((int64_t)a.H * nW[m]), 256, 0, st>>>(outW[m], dW[m], nW[m], a.B, a.H, 1);
      x.check(cudaGetLastError());
    }
  }
  if (cudaFreeAsync(base, st) != cudaSuccess) x.ok = false;
  return x.ok ? TTT_OK : TTT_ERR_CUDA;
}

}  // namespace ttt
