// LaCT SwiGLU fast-weight layer forward ("Test-Time Training Done Right"
// review, sections 3.2-3.3 and 4 / Figure 3).
//
// Per (batch, head) z the fast weights W1, W3 [dh][dk] and W2 [dv][dh] live
// in fp32 master copies in scratch memory, with bf16 operand copies refreshed
// after every update (W1 and W3 rows interleaved in blocks of 64 into W13 so
// that 128 consecutive W13 rows give matching h1/h3 columns). One chunk step,
// all heads at once (causal order: apply with the weights before the chunk,
// then update):
//   L1  Aq = silu(Q W1^T) * (Q W3^T)         [b x dh] bf16          (causal)
//       per 128 tokens x 64 hidden units, one accumulator tile holds
//       H1 | H3 = K [W1;W3]^T and U = V W2 for those units; with Gz = -eta U:
//       Ak' = eta silu(H1) H3, dH3 = Gz silu(H1), dH1 = Gz H3 silu'(H1)
//                                            [b x dh] bf16 (Gz never leaves TMEM)
//   L2  Y  = Aq W2^T -> layer output         [b x dv]               (causal)
//       G1 = dH1^T K, G3 = dH3^T K           [dh x dk] fp32 (split-K, TMA add)
//       G2 = -V^T Ak'                        [dv x dh]
//   L3  Muon: G <- NS5(G) (split-bf16 tensor-core MMAs, fp32 accumulation)
//   L4  W <- W - G; each row rescaled to its initial L2 norm; bf16 copies.
// Non-causal (update, then apply): L1 without Aq, L2 without Y, L3, L4, then
// Aq and Y with the updated weights.
// Precision: GD uses bf16 operands with fp32 accumulation; Muon uses
// split-bf16 operands (x = hi + lo, products hi*hi + lo*hi + hi*lo) on the
// update path because the unit-step Muon scan amplifies per-chunk rounding
// across chunks. The apply path (Aq, Y) feeds only the output: there the
// weights keep hi / lo and Aq is plain bf16.
#include <cooperative_groups.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>

#include "gemm_tc.cuh"
#include "lact.cuh"

namespace ttt {
namespace {

using gemm::Operand;
using gemm::Params;
using gemm::Problem;

constexpr int BN = 256;     // GEMM tile width (W13 interleave block = BN / 2)

// ---------------------------------------------------------------------------
// Row kernels: prepare / update / renormalise the fast weights
// ---------------------------------------------------------------------------

struct RowArgs {
  float* Wm[3];            // masters: W1 [Z][dh][dk], W3 [Z][dh][dk], W2 [Z][dv][dh]
  const float* Win[3];     // inputs (prep only), per-head or per-(batch, head)
  int64_t win_sz[3];       // non-zero when the input holds one matrix per (batch, head)
  float* rho[3];           // initial row norms [Z][rows]
  float* G[3];             // gradients (update input; zeroed after use)
  __nv_bfloat16 *w13_hi, *w13_lo, *w2_hi, *w2_lo;
  int Z, H, dk, dv, dh;
  int prep;                // 1: copy inputs and record norms; 0: W -= G then renorm
  int split;
  // momentum (same row order): M <- beta M + G, then W -= M instead of W -= G
  int momentum;
  float beta;
  float* M[3];             // momentum masters [Z][rows][cols]
  const float* Min[3];     // initial momentum (prep only; null: zero)
  int64_t min_sz[3];       // non-zero when Min holds one matrix per (batch, head)
  int* status;             // device status word (index checks of the debug-bounds build)
};

// One warp per (z, row of W1 | W3 | W2).
__global__ void __launch_bounds__(256) lact_rows_kernel(RowArgs a) {
  pdl_wait();
  pdl_trigger();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int rows_z = 2 * a.dh + a.dv;
  if (gw >= a.Z * rows_z) return;
  const int z = gw / rows_z;
  int r = gw % rows_z, m;
  if (r < a.dh) {
    m = 0;
  } else if (r < 2 * a.dh) {
    m = 1;
    r -= a.dh;
  } else {
    m = 2;
    r -= 2 * a.dh;
  }
  const int len = (m == 2) ? a.dh : a.dk;
  const int nrows = (m == 2) ? a.dv : a.dh;
  float* W = a.Wm[m] + ((int64_t)z * nrows + r) * len;
  float* G = a.G[m] + ((int64_t)z * nrows + r) * len;
  const float* src = nullptr;
  if (a.prep) {
    const int zin = a.win_sz[m] ? z : z % a.H;
    src = a.Win[m] + ((int64_t)zin * nrows + r) * len;
  }
  float* rho = a.rho[m] + (int64_t)z * nrows + r;
  float* M = a.momentum ? a.M[m] + ((int64_t)z * nrows + r) * len : nullptr;
  const float* msrc = nullptr;
  if (a.prep && a.momentum && a.Min[m]) {
    const int zin = a.min_sz[m] ? z : z % a.H;
    msrc = a.Min[m] + ((int64_t)zin * nrows + r) * len;
  }
  __nv_bfloat16 *hi, *lo;
  int64_t orow;
  if (m == 2) {
    hi = a.w2_hi;
    lo = a.w2_lo;
    orow = (int64_t)z * a.dv + r;
  } else {
    hi = a.w13_hi;
    lo = a.w13_lo;
    orow = (int64_t)z * 2 * a.dh + (r / gemm::kHid) * 2 * gemm::kHid + (m == 1 ? gemm::kHid : 0) +
           (r % gemm::kHid);
  }
  if (!TTT_BOUNDS(orow >= 0 && orow < (int64_t)a.Z * (m == 2 ? a.dv : 2 * a.dh) && r < nrows &&
                      (len % 128 != 0 || len <= 1024),
                  a.status))
    return;
  hi += orow * len;
  if (a.split) lo += orow * len;

  // new row = (W - G) (or the input row), then rescaled to its initial norm
  auto finish = [&](float ss, float& s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float nrm = sqrtf(ss);
    if (a.prep) {
      if (lane == 0) *rho = nrm;
      s = 1.f;
    } else {
      const float target = *rho;
      s = nrm > 0.f ? target / nrm : 1.f;
    }
  };
  if (len % 128 == 0) {
    // 4 consecutive columns per lane: 16-byte loads and stores, all issued
    // before the row reduction
    constexpr int kMaxV = 8;  // len <= 1024
    const int per = len / 128;
    float4 v[kMaxV];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxV; ++i) {
      if (i >= per) break;
      const int c = 4 * (lane + 32 * i);
      if (a.prep) {
        v[i] = *reinterpret_cast<const float4*>(src + c);
        if (M)
          *reinterpret_cast<float4*>(M + c) =
              msrc ? *reinterpret_cast<const float4*>(msrc + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const float4 w = *reinterpret_cast<const float4*>(W + c);
        float4 g = *reinterpret_cast<const float4*>(G + c);
        if (M) {  // heavy-ball momentum: the step is beta * M + G
          const float4 mo = *reinterpret_cast<const float4*>(M + c);
          g = make_float4(fmaf(a.beta, mo.x, g.x), fmaf(a.beta, mo.y, g.y), fmaf(a.beta, mo.z, g.z),
                          fmaf(a.beta, mo.w, g.w));
          *reinterpret_cast<float4*>(M + c) = g;
        }
        v[i] = make_float4(w.x - g.x, w.y - g.y, w.z - g.z, w.w - g.w);
      }
      ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    }
    float s;
    finish(ss, s);
#pragma unroll
    for (int i = 0; i < kMaxV; ++i) {
      if (i >= per) break;
      const int c = 4 * (lane + 32 * i);
      const float4 x = make_float4(v[i].x * s, v[i].y * s, v[i].z * s, v[i].w * s);
      *reinterpret_cast<float4*>(W + c) = x;
      *reinterpret_cast<float4*>(G + c) = make_float4(0.f, 0.f, 0.f, 0.f);
      uint32_t h0, h1, l0, l1;
      gemm::split_bf16x2(x.x, x.y, h0, l0);
      gemm::split_bf16x2(x.z, x.w, h1, l1);
      *reinterpret_cast<uint2*>(hi + c) = make_uint2(h0, h1);
      if (a.split) *reinterpret_cast<uint2*>(lo + c) = make_uint2(l0, l1);
    }
    return;
  }
  // rows of 32 or 64 columns: one value per lane per step
  float v[2];
  float ss = 0.f;
  const int per = len / 32;  // 1 or 2: the supported sizes give len 64 or a multiple of 128
  if (per > 2) return;
  for (int i = 0; i < per; ++i) {
    const int c = lane + 32 * i;
    if (a.prep) {
      v[i] = src[c];
      if (M) M[c] = msrc ? msrc[c] : 0.f;
    } else {
      float g = G[c];
      if (M) {
        g = fmaf(a.beta, M[c], g);
        M[c] = g;
      }
      v[i] = W[c] - g;
    }
    ss += v[i] * v[i];
  }
  float s;
  finish(ss, s);
  for (int i = 0; i < per; ++i) {
    const int c = lane + 32 * i;
    const float x = v[i] * s;
    W[c] = x;
    G[c] = 0.f;
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[c] = h;
    if (a.split) lo[c] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

// ---------------------------------------------------------------------------
// Newton-Schulz (Muon) on the tensor cores in split-bf16 precision: a cluster
// of kNsCluster CTAs per gradient matrix, each owning one slab of the long
// side. Gram partials meet in L2-resident scratch between cluster barriers;
// every CTA then forms the (small) polynomial itself and updates its slab.
// ---------------------------------------------------------------------------

constexpr int kNsCluster = 4;

struct NsArgs {
  float* G[3];   // in/out, [Z][rows][cols] row-major
  int rows[3], cols[3];
  // per (z, m), s = min(rows, cols), L = max(rows, cols) / kNsCluster:
  // Gram partials [2][kNsCluster][s*s], then per CTA gram [s*s], poly [s*s],
  // xn [L*s], then kNsCluster partial squared norms
  float* scratch;
  int64_t scratch_stride;
  int* status;  // device status word (bounded waits record a timeout here)
  float a, b, c, eps;
  int steps;
};

constexpr int kNsThreads = 1024;

// C[M x N] = alpha * op(A) op(B) + beta * Cin, all row-major fp32 in global
// memory (L2-resident scratch; row strides lda, ldb, ldc and ldcin); op(A) is
// A or A^T (tA), same for B. Computed
// by the whole CTA (32 warps) on the tensor cores with m16n8k16 MMAs in
// split-bf16 precision: each fp32 operand x is held as hi = bf16(x) and
// lo = bf16(x - hi), and the product accumulates hi*hi + lo*hi + hi*lo in fp32
// (relative error about 2^-16 per product, near fp32). Output tiles are
// 128 x 128; warp (wm, wn) of a 4 x 8 grid owns rows 32*wm.., columns 16*wn...
constexpr int kNsTM = 128, kNsTN = 128, kNsTK = 32;
constexpr int kNsLdA = kNsTK + 8;   // padded row length (bf16) of the A tiles
constexpr int kNsLdB = kNsTN + 8;   // padded row length (bf16) of the B tiles

__device__ __forceinline__ void ns_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ns_ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void ns_ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

__device__ void cta_gemm(float* C, const float* Cin, const float* A, const float* B, int M, int N,
                         int K, bool tA, bool tB, int lda, int ldb, int ldc, int ldcin,
                         float alpha, float beta) {
  __shared__ __align__(16) __nv_bfloat16 sa[2][kNsTM * kNsLdA];  // [hi|lo][m][k]
  __shared__ __align__(16) __nv_bfloat16 sb[2][kNsTK * kNsLdB];  // [hi|lo][k][n]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 3, wn = warp & 7;
  const int mi = lane >> 3, rr = lane & 7, g = lane >> 2, c4 = lane & 3;
  for (int i0 = 0; i0 < M; i0 += kNsTM)
    for (int j0 = 0; j0 < N; j0 += kNsTN) {
      float acc[2][2][4] = {};
      for (int k0 = 0; k0 < K; k0 += kNsTK) {
        // A tile [128 x 32] and B tile [32 x 128]: fp32 -> bf16 hi / lo
        for (int e = tid; e < kNsTM * kNsTK; e += kNsThreads) {
          int m, k;
          if (tA) { m = e % kNsTM; k = e / kNsTM; } else { m = e / kNsTK; k = e % kNsTK; }
          const int gi = i0 + m, gk = k0 + k;
          float x = 0.f;
          if (gi < M && gk < K) x = tA ? A[(int64_t)gk * lda + gi] : A[(int64_t)gi * lda + gk];
          const __nv_bfloat16 h = __float2bfloat16_rn(x);
          sa[0][m * kNsLdA + k] = h;
          sa[1][m * kNsLdA + k] = __float2bfloat16_rn(x - __bfloat162float(h));
        }
        for (int e = tid; e < kNsTK * kNsTN; e += kNsThreads) {
          int k, n;
          if (tB) { k = e % kNsTK; n = e / kNsTK; } else { k = e / kNsTN; n = e % kNsTN; }
          const int gk = k0 + k, gj = j0 + n;
          float x = 0.f;
          if (gk < K && gj < N) x = tB ? B[(int64_t)gj * ldb + gk] : B[(int64_t)gk * ldb + gj];
          const __nv_bfloat16 h = __float2bfloat16_rn(x);
          sb[0][k * kNsLdB + n] = h;
          sb[1][k * kNsLdB + n] = __float2bfloat16_rn(x - __bfloat162float(h));
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kNsTK; kk += 16) {
          uint32_t af[2][2][4], bf[2][2][2];  // [hi|lo][m or n tile]
#pragma unroll
          for (int x = 0; x < 2; ++x) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
              ns_ldsm_x4(af[x][mt], &sa[x][(32 * wm + 16 * mt + rr + 8 * (mi & 1)) * kNsLdA + kk +
                                           8 * (mi >> 1)]);
            uint32_t r[4];
            ns_ldsm_x4_t(r, &sb[x][(kk + rr + 8 * (mi & 1)) * kNsLdB + 16 * wn + 8 * (mi >> 1)]);
            bf[x][0][0] = r[0];
            bf[x][0][1] = r[1];
            bf[x][1][0] = r[2];
            bf[x][1][1] = r[3];
          }
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              ns_mma(acc[mt][nt], af[0][mt], bf[0][nt][0], bf[0][nt][1]);  // hi * hi
              ns_mma(acc[mt][nt], af[1][mt], bf[0][nt][0], bf[0][nt][1]);  // lo * hi
              ns_mma(acc[mt][nt], af[0][mt], bf[1][nt][0], bf[1][nt][1]);  // hi * lo
            }
        }
        __syncthreads();
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = i0 + 32 * wm + 16 * mt + g + 8 * (q >> 1);
            const int j = j0 + 16 * wn + 8 * nt + 2 * c4 + (q & 1);
            if (i < M && j < N) {
              const float prev = (beta != 0.f) ? Cin[(int64_t)i * ldcin + j] : 0.f;
              C[(int64_t)i * ldc + j] = alpha * acc[mt][nt][q] + beta * prev;
            }
          }
      __syncthreads();
    }
}

__device__ __forceinline__ void cluster_sync_all() {
  __threadfence();
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ float block_sum(float v) {
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
  return t;
}

// X <- NS5(X / (||X||_F + eps)). Tall X (rows >= cols): X <- a X + X (b A + c A^2)
// with A = X^T X; wide X: X <- a X + (b A + c A^2) X with A = X X^T. CTA c of
// the cluster owns rows (tall) or columns (wide) [c L, c L + L) of X.
__global__ void __cluster_dims__(kNsCluster, 1, 1) __launch_bounds__(kNsThreads)
    ns_kernel(NsArgs a) {
  pdl_wait();
  pdl_trigger();
  const int mat = blockIdx.x / kNsCluster, c = blockIdx.x % kNsCluster;
  const int z = mat / 3, m = mat % 3;
  const int R = a.rows[m], C = a.cols[m];
  float* X = a.G[m] + (int64_t)z * R * C;
  const bool tall = R >= C;
  const int s = tall ? C : R;
  const int L = (tall ? R : C) / kNsCluster;
  float* Xc = tall ? X + (int64_t)c * L * C : X + (int64_t)c * L;  // row stride C
  float* base = a.scratch + (int64_t)mat * a.scratch_stride;
  float* parts = base;
  float* gram = parts + 2 * kNsCluster * s * s + (int64_t)c * (2 * s * s + L * s);
  float* poly = gram + (int64_t)s * s;
  float* xn = poly + (int64_t)s * s;
  float* nrm = base + 2 * kNsCluster * s * s + (int64_t)kNsCluster * (2 * s * s + L * s);
  const int sr = tall ? L : s, sc = tall ? s : L;  // slab rows x columns (row stride C)
  const int tid = threadIdx.x;

  float ss = 0.f;
  for (int e = tid; e < sr * sc; e += kNsThreads) {
    const float x = Xc[(int64_t)(e / sc) * C + e % sc];
    ss += x * x;
  }
  ss = block_sum(ss);
  if (tid == 0) nrm[c] = ss;
  cluster_sync_all();
  float tot = 0.f;
  for (int i = 0; i < kNsCluster; ++i) tot += __ldcg(nrm + i);  // other CTAs' writes: bypass L1
  const float inv = 1.f / (sqrtf(tot) + a.eps);
  for (int e = tid; e < sr * sc; e += kNsThreads) Xc[(int64_t)(e / sc) * C + e % sc] *= inv;
  __syncthreads();
  for (int it = 0; it < a.steps; ++it) {
    float* part = parts + ((int64_t)(it & 1) * kNsCluster + c) * s * s;
    if (tall)
      cta_gemm(part, nullptr, Xc, Xc, s, s, L, true, false, C, C, s, s, 1.f, 0.f);
    else
      cta_gemm(part, nullptr, Xc, Xc, s, s, L, false, true, C, C, s, s, 1.f, 0.f);
    cluster_sync_all();
    const float* pb = parts + (int64_t)(it & 1) * kNsCluster * s * s;
    for (int e = tid; e < s * s; e += kNsThreads) {
      float g = 0.f;
      for (int i = 0; i < kNsCluster; ++i) g += __ldcg(pb + (int64_t)i * s * s + e);
      gram[e] = g;
    }
    __syncthreads();
    // poly = c gram^2 + b gram
    cta_gemm(poly, gram, gram, gram, s, s, s, false, false, s, s, s, s, a.c, a.b);
    // xn = slab poly (tall) or poly slab (wide), plus a * slab
    if (tall)
      cta_gemm(xn, Xc, Xc, poly, L, s, s, false, false, C, s, s, C, 1.f, a.a);
    else
      cta_gemm(xn, Xc, poly, Xc, s, L, s, false, false, s, C, L, C, 1.f, a.a);
    for (int e = tid; e < sr * sc; e += kNsThreads)
      Xc[(int64_t)(e / sc) * C + e % sc] = xn[e];
    __syncthreads();
  }
}

constexpr int kN5 = 128;          // slab side of the 128 x 512 Newton-Schulz kernel

// ---------------------------------------------------------------------------
// Newton-Schulz for 128 x 512 (or 512 x 128) gradients on the 5th-generation
// tensor cores: a cluster of kNsCluster CTAs per matrix, CTA c owning the
// 128 x 128 slab c of the long side. The Gram matrix M = X^T X of the
// normalised gradient is formed once: partials over the slabs are summed
// through distributed shared memory (CTA c reduces rows [32c, 32c + 32) and
// writes them into every CTA's copy). The five iterations then run on the
// Gram side with no further exchange: a X + b (X X^T) X + c (X X^T)^2 X equals
// X P with P = a I + b M + c M^2, which commutes with M, so the next Gram
// matrix is P M P; each CTA updates its own slab and its own copy of M (four
// 128 x 128 products per iteration). X, M and P stay in shared memory as bf16 hi / lo
// (x = hi + lo to about 16 bits) in the 128-byte-swizzled layout of two
// 64-column boxes [128 rows][128 B]; one storage serves as a K-major operand
// (rows = M or N) and as an MN-major operand (rows = K). Each split product
// hi*hi + lo*hi + hi*lo is 24 tcgen05.mma of 128 x 128 x 16 into one TMEM
// accumulator, issued by one thread; 16 warps move accumulators out of TMEM.
// ---------------------------------------------------------------------------

constexpr int kT5Threads = 512;
constexpr uint32_t kT5Box = 16384;  // one 64-column box of a 128 x 128 bf16 matrix

struct Ns5Smem {
  alignas(1024) uint8_t x[2][2 * kT5Box];  // [hi|lo]
  alignas(1024) uint8_t g[2][2 * kT5Box];
  alignas(1024) uint8_t p[2][2 * kT5Box];  // also the fp32 Gram partial [128][128]
  uint64_t mma_done[2];  // one per TMEM accumulator
  uint32_t tmem_base;
  float nrm;
};

// byte offset of bf16 element (r, c) of a 128 x 128 matrix in the box layout
__device__ __forceinline__ uint32_t t5_off(int r, int c) {
  return (uint32_t)((c >> 6) * kT5Box + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) +
                    ((c & 7) << 1));
}
// byte offset of 16-byte fp32 chunk j (columns 4j .. 4j+3) of row r of the partial
__device__ __forceinline__ uint32_t t5_part(int r, int j) {
  return (uint32_t)(r * 512 + ((j ^ (r & 7)) << 4));
}

__global__ void __cluster_dims__(kNsCluster, 1, 1) __launch_bounds__(kT5Threads, 1)
    ns5_kernel(NsArgs a) {
  extern __shared__ __align__(1024) uint8_t ns5_raw[];
  Ns5Smem& sm = *reinterpret_cast<Ns5Smem*>((reinterpret_cast<uintptr_t>(ns5_raw) + 1023) &
                                            ~uintptr_t(1023));
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int mat = blockIdx.x / kNsCluster, c = (int)cluster.block_rank();
  const int z = mat / 3, m = mat % 3;
  const int R = a.rows[m], C = a.cols[m];
  const bool tall = R >= C;
  float* Xc = a.G[m] + (int64_t)z * R * C + (tall ? (int64_t)c * kN5 * C : (int64_t)c * kN5);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this CTA's 128 x 128 slab lies inside the matrix (a failed check skips the
  // slab's global loads and stores but keeps every cluster barrier)
  const bool slab_ok = TTT_BOUNDS(tall ? (C == kN5 && (c + 1) * kN5 <= R)
                                       : (R == kN5 && (c + 1) * kN5 <= C),
                                  a.status);

  if (tid == 0) {
    mbar_init(&sm.mma_done[0], 1);
    mbar_init(&sm.mma_done[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) umma::tmem_alloc(&sm.tmem_base, 256);  // two 128-column accumulators
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();
  pdl_trigger();

  // Frobenius norm of the whole matrix (four slabs), then the scaled slab as hi / lo
  // the slab as 8-column pieces (two float4 each), 4 per thread, kept in registers
  float4 xs[4][2];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + i * kT5Threads, r = e >> 4, c0 = (e & 15) * 8;
    const float4* src = reinterpret_cast<const float4*>(Xc + (int64_t)r * C + c0);
    xs[i][0] = slab_ok ? src[0] : make_float4(0.f, 0.f, 0.f, 0.f);
    xs[i][1] = slab_ok ? src[1] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += xs[i][0].x * xs[i][0].x + xs[i][0].y * xs[i][0].y + xs[i][0].z * xs[i][0].z +
          xs[i][0].w * xs[i][0].w + xs[i][1].x * xs[i][1].x + xs[i][1].y * xs[i][1].y +
          xs[i][1].z * xs[i][1].z + xs[i][1].w * xs[i][1].w;
  }
  ss = block_sum(ss);
  if (tid == 0) sm.nrm = ss;
  cluster.sync();
  float tot = 0.f;
  for (int r = 0; r < kNsCluster; ++r) tot += *cluster.map_shared_rank(&sm.nrm, r);
  const float inv = 1.f / (sqrtf(tot) + a.eps);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + i * kT5Threads, r = e >> 4, c0 = (e & 15) * 8;
    const float xv[8] = {xs[i][0].x, xs[i][0].y, xs[i][0].z, xs[i][0].w,
                         xs[i][1].x, xs[i][1].y, xs[i][1].z, xs[i][1].w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      gemm::split_bf16x2(xv[2 * u] * inv, xv[2 * u + 1] * inv, hi[u], lo[u]);
    }
    *reinterpret_cast<uint4*>(sm.x[0] + t5_off(r, c0)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(sm.x[1] + t5_off(r, c0)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  umma::fence_proxy_async_smem();
  __syncthreads();

  // One split product into accumulator `acc` (0 or 1): A, B given as [hi, lo]
  // storages and whether each is read MN-major (rows = K) or K-major (rows =
  // M or N). issue() enqueues the 24 MMAs from one thread and commits them to
  // the accumulator's barrier; wait() blocks every thread until they are done.
  int phase[2] = {0, 0};
  auto issue = [&](uint8_t* const (&A)[2], bool a_mn, uint8_t* const (&B)[2], bool b_mn, int acc) {
    if (tid == 0) {
      umma::fence_after();
      const uint32_t idesc = umma::instr_desc(1, kN5, kN5, a_mn, b_mn);
      const int pa[3] = {0, 1, 0}, pb[3] = {0, 0, 1};
      for (int pr = 0; pr < 3; ++pr) {
        const uint32_t sa = smem_u32(A[pa[pr]]), sb = smem_u32(B[pb[pr]]);
#pragma unroll
        for (int kk = 0; kk < kN5 / 16; ++kk) {
          const uint64_t ad = a_mn ? umma::smem_desc(sa + kk * 2048, kT5Box, 1024)
                                   : umma::smem_desc(sa + (kk >> 2) * kT5Box + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = b_mn ? umma::smem_desc(sb + kk * 2048, kT5Box, 1024)
                                   : umma::smem_desc(sb + (kk >> 2) * kT5Box + (kk & 3) * 32, 16, 1024);
          umma::mma_bf16(tmem + 128 * acc, ad, bd, idesc, (pr > 0 || kk > 0) ? 1u : 0u);
        }
      }
      umma::commit(&sm.mma_done[acc]);
    }
  };
  auto wait = [&](int acc) {
    const bool ok = mbar_wait(&sm.mma_done[acc], phase[acc], a.status);
    phase[acc] ^= 1;
    umma::fence_after();
    return ok;
  };
  auto product = [&](uint8_t* const (&A)[2], bool a_mn, uint8_t* const (&B)[2], bool b_mn) {
    issue(A, a_mn, B, b_mn, 0);
    return wait(0);
  };
  // This thread's 32 accumulator values: row 32 (warp & 3) + lane, columns 32 (warp >> 2) ..
  const int er = 32 * (warp & 3) + lane, ec = 32 * (warp >> 2);
  const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + ec;
  auto acc_load = [&](float (&v)[32], int acc = 0) {
    uint32_t r0[16], r1[16];
    umma::tmem_ld16_async(tl + 128 * acc, r0);
    umma::tmem_ld16_async(tl + 128 * acc + 16, r1);
    umma::tmem_wait_ld(r0);
    umma::tmem_wait_ld(r1);
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = __uint_as_float(r0[u]), v[16 + u] = __uint_as_float(r1[u]);
  };
  // values (hi + lo) of bf16 storage elements (r, cc .. cc+31), 16-byte reads
  auto val32 = [&](uint8_t* const (&S)[2], int r, int cc, float (&o)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 h = *reinterpret_cast<const uint4*>(S[0] + t5_off(r, cc + 8 * q));
      const uint4 l = *reinterpret_cast<const uint4*>(S[1] + t5_off(r, cc + 8 * q));
      const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162*>(&hw[u]);
        const __nv_bfloat162 lb = *reinterpret_cast<const __nv_bfloat162*>(&lw[u]);
        o[8 * q + 2 * u] = __low2float(hb) + __low2float(lb);
        o[8 * q + 2 * u + 1] = __high2float(hb) + __high2float(lb);
      }
    }
  };
  // store 32 values of row r, columns cc .. cc+31, as hi / lo
  auto put32 = [&](uint8_t* const (&S)[2], int r, int cc, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        gemm::split_bf16x2(v[8 * q + 2 * u], v[8 * q + 2 * u + 1], hi[u], lo[u]);
      }
      *reinterpret_cast<uint4*>(S[0] + t5_off(r, cc + 8 * q)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(S[1] + t5_off(r, cc + 8 * q)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  };

  uint8_t* const X2[2] = {sm.x[0], sm.x[1]};
  uint8_t* const G2[2] = {sm.g[0], sm.g[1]};
  uint8_t* const P2[2] = {sm.p[0], sm.p[1]};
  uint8_t* const part = sm.p[0];  // 64 KB: p[0] and p[1] are contiguous
  bool ok = true;
  // The Gram matrix of the whole (normalised) X, once: partial over this
  // CTA's slab (tall X^T X, both operands MN-major; wide X X^T, both
  // K-major), then CTA c sums rows [32c, 32c + 32) of the four partials and
  // writes them into every CTA's M (sm.g) as hi / lo.
  ok = product(X2, tall, X2, tall) && ok;
  {
    float v[32];
    acc_load(v);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *reinterpret_cast<float4*>(part + t5_part(er, ec / 4 + q)) =
          make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  }
  umma::fence_before();
  cluster.sync();
  {
    const int r = 32 * c + (tid >> 4), c0 = (tid & 15) * 8;
    float gsum[8] = {};
    for (int rk = 0; rk < kNsCluster; ++rk) {
      const uint8_t* rp = cluster.map_shared_rank(part, rk);
      const float4 u0 = *reinterpret_cast<const float4*>(rp + t5_part(r, c0 / 4));
      const float4 u1 = *reinterpret_cast<const float4*>(rp + t5_part(r, c0 / 4 + 1));
      gsum[0] += u0.x, gsum[1] += u0.y, gsum[2] += u0.z, gsum[3] += u0.w;
      gsum[4] += u1.x, gsum[5] += u1.y, gsum[6] += u1.z, gsum[7] += u1.w;
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      gemm::split_bf16x2(gsum[2 * u], gsum[2 * u + 1], hi[u], lo[u]);
    }
    for (int rk = 0; rk < kNsCluster; ++rk) {
      *reinterpret_cast<uint4*>(cluster.map_shared_rank(sm.g[0], rk) + t5_off(r, c0)) =
          make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(cluster.map_shared_rank(sm.g[1], rk) + t5_off(r, c0)) =
          make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  cluster.sync();
  umma::fence_proxy_async_smem();
  __syncthreads();
  // The iteration on the Gram side, with no further exchange: with
  // P = a I + b M + c M^2 (a polynomial in M = X^T X, so symmetric and
  // commuting with M), a X + b (X X^T) X + c (X X^T)^2 X = X P, and the next
  // Gram matrix is (X P)^T (X P) = P M P. Each CTA updates its own slab
  // (X <- X P tall, P X wide) and its own copy of M.
  auto sync_operands = [&]() {
    umma::fence_before();
    umma::fence_proxy_async_smem();
    __syncthreads();
  };
  for (int it = 0; it < a.steps; ++it) {
    // P = a I + b M + c M^2
    ok = product(G2, false, G2, true) && ok;
    {
      float v[32], gv[32];
      acc_load(v);
      val32(G2, er, ec, gv);
#pragma unroll
      for (int u = 0; u < 32; ++u) v[u] = a.c * v[u] + a.b * gv[u] + (ec + u == er ? a.a : 0.f);
      put32(P2, er, ec, v);
    }
    sync_operands();
    // X <- X P (tall) or P X (wide)   (B MN-major) into accumulator 0, and,
    // unless this is the last step, T = M P into accumulator 1 right behind it:
    // the X epilogue then overlaps the M P products.
    const bool last = it + 1 == a.steps;
    if (tall)
      issue(X2, false, P2, true, 0);
    else
      issue(P2, false, X2, true, 0);
    if (!last) issue(G2, false, P2, true, 1);
    ok = wait(0) && ok;
    {
      float v[32];
      acc_load(v, 0);
      if (last) {
        float4* dst = reinterpret_cast<float4*>(Xc + (int64_t)er * C + ec);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (slab_ok) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        put32(X2, er, ec, v);
      }
    }
    if (last) break;
    // M <- P (M P): T = M P (accumulator 1) into M's storage, then P T
    ok = wait(1) && ok;
    {
      float v[32];
      acc_load(v, 1);
      put32(G2, er, ec, v);
    }
    sync_operands();
    ok = product(P2, false, G2, true) && ok;
    {
      float v[32];
      acc_load(v);
      put32(G2, er, ec, v);
    }
    sync_operands();
    // A timed-out wait is recorded in the status word; the loop still runs to
    // its end so that every CTA of the cluster meets the same cluster barriers.
  }
  (void)ok;
  cluster.sync();  // no CTA leaves while another may still read its shared memory
  if (warp == 0) umma::tmem_dealloc(tmem, 256);
}

__global__ void copy_kernel(float* dst, const float* src, int64_t n) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

bool map_tokens(CUtensorMap* m, const TokView& v, int B, int H, int T, int d, int box_inner,
                int box_rows) {
  TokView x = v;
  if (B == 1) x.sb = (int64_t)H * T * d;
  if (H == 1) x.sh = (int64_t)T * d;
  if (T == 1) x.st = d;
  uint64_t dims[4] = {(uint64_t)d, (uint64_t)T, (uint64_t)H, (uint64_t)B};
  uint64_t strides[3] = {(uint64_t)x.st * 2, (uint64_t)x.sh * 2, (uint64_t)x.sb * 2};
  uint32_t box[4] = {(uint32_t)box_inner, (uint32_t)box_rows, 1, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x.p, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

// [Z][rows_alloc][cols] bf16 buffer as a 4-d map {cols, rows, Z, 1}; only the
// first `rows` rows of each z are visible (later rows read as zeros).
bool map_buf(CUtensorMap* m, const void* base, int Z, int rows, int rows_alloc, int cols,
             int box_inner, int box_rows) {
  uint64_t dims[4] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)Z, 1};
  uint64_t strides[3] = {(uint64_t)cols * 2, (uint64_t)cols * 2 * rows_alloc,
                         (uint64_t)cols * 2 * rows_alloc * Z};
  uint32_t box[4] = {(uint32_t)box_inner, (uint32_t)box_rows, 1, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

// fp32 gradient [Z][rows][cols] as a TMA add-reduction target: box of
// {32 columns, 32 rows} (128-byte rows) with the 128-byte swizzle of the
// epilogue's staging buffers.
bool grad_map(CUtensorMap* m, const float* base, int Z, int rows, int cols) {
  uint64_t dims[4] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)Z, 1};
  uint64_t strides[3] = {(uint64_t)cols * 4, (uint64_t)cols * 4 * rows,
                         (uint64_t)cols * 4 * rows * Z};
  uint32_t box[4] = {32, 32, 1, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

struct Scratch {
  float *Wm[3], *rho[3], *G[3], *ns, *M[3];
  __nv_bfloat16 *w13[2], *w2[2];          // hi, lo
  __nv_bfloat16 *aq[2], *ak[2], *dh1[2], *dh3[2];
  int64_t ns_stride;
};

void fill_problem_tiles(Params& P) {
  int t = 0;
  for (int i = 0; i < P.nprob; ++i) {
    Problem& p = P.p[i];
    p.mtiles = (p.M + gemm::BM - 1) / gemm::BM;
    p.ntiles = (p.N + p.tn - 1) / p.tn;
    p.tile_begin = t;
    p.kblocks = (p.K + gemm::BK - 1) / gemm::BK;
    p.kb_per = (p.kblocks + p.ksplit - 1) / p.ksplit;
    auto mag = [](int d) { return ((uint64_t(1) << 32) + (uint64_t)d - 1) / (uint64_t)d; };
    p.mag_n = mag(p.ntiles);
    p.mag_m = mag(p.mtiles);
    p.mag_k = mag(p.ksplit);
    t += p.nz * p.ksplit * p.mtiles * p.ntiles;
  }
  P.total_tiles = t;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = 148;
  }
  return n;
}

// Persistent launch: one CTA per SM (or fewer if there are fewer tiles).
// The dynamic shared-memory limit of the GEMM kernel is raised once per device.
cudaError_t gemm_attr_once() {
  constexpr int kMaxDevices = 64;
  static bool done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < kMaxDevices && done[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gemm::gemm_kernel<BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(sizeof(gemm::Smem<BN>) + 1024));
  if (e == cudaSuccess && dev < kMaxDevices) done[dev] = true;
  return e;
}

cudaError_t launch_gemm(Params& P, cudaStream_t s) {
  fill_problem_tiles(P);
  if (P.total_tiles == 0) return cudaSuccess;
  const size_t smem = sizeof(gemm::Smem<BN>) + 1024;
  cudaError_t e = gemm_attr_once();
  if (e != cudaSuccess) return e;
  const int grid = P.total_tiles < num_sms() ? P.total_tiles : num_sms();
  return launch_pdl(gemm::gemm_kernel<BN>, dim3(grid), dim3(gemm::kThreads), smem, s, P);
}

// Operand helpers -----------------------------------------------------------
// K-major token operand (rows = tokens of the chunk): storage [T][d].
bool tok_kmajor(Operand& o, const TokView& v, const LactArgs& a, int d, int row0, int box_rows) {
  o.mn_major = 0;
  o.row0 = row0;
  o.zdiv = a.H;
  return map_tokens(&o.map[0], v, a.B, a.H, a.T, d, 64, box_rows) &&
         map_tokens(&o.map[1], v, a.B, a.H, a.T, d, 64, box_rows);
}
// MN-major token operand (tokens = K dimension): storage [T][d], d = M or N.
bool tok_mnmajor(Operand& o, const TokView& v, const LactArgs& a, int d, int row0) {
  o.mn_major = 1;
  o.row0 = row0;
  o.zdiv = a.H;
  return map_tokens(&o.map[0], v, a.B, a.H, a.T, d, 64, 64) &&
         map_tokens(&o.map[1], v, a.B, a.H, a.T, d, 64, 64);
}
bool buf_op(Operand& o, __nv_bfloat16* const* hl, int Z, int rows, int rows_alloc, int cols,
            int mn_major, int box_rows, bool split) {
  o.mn_major = mn_major;
  o.row0 = 0;
  o.zdiv = Z;
  const int br = mn_major ? 64 : box_rows;
  return map_buf(&o.map[0], hl[0], Z, rows, rows_alloc, cols, 64, br) &&
         map_buf(&o.map[1], split ? hl[1] : hl[0], Z, rows, rows_alloc, cols, 64, br);
}

void segs(Problem& p, int n, const int (*ab)[2]) {
  p.nseg = n;
  for (int i = 0; i < n; ++i) {
    p.seg_a[i] = ab[i][0];
    p.seg_b[i] = ab[i][1];
  }
}
const int kSegExact[1][2] = {{0, 0}};
const int kSegBsplit[2][2] = {{0, 0}, {0, 1}};
const int kSegAsplit[2][2] = {{0, 0}, {1, 0}};

gemm::EpiArgs epi_base(const LactArgs& a, int s0, int rows_valid) {
  gemm::EpiArgs e;
  memset(&e, 0, sizeof(e));
  e.eta = a.eta;
  e.eta_t0 = s0;
  e.H = a.H;
  e.out = a.out;
  e.out_bf16 = a.dtype == TTT_BF16;
  e.rows_valid = rows_valid;
  e.scale = 1.f;
  e.nsplit = 1;
  e.ozdiv = 1;
  return e;
}

// Split the token reduction so that the gradient GEMMs give about two tiles
// per SM, but keep at least 4 K blocks per split.
int pick_ksplit(int kblocks, int tiles) {
  int ks = 1;
  while (ks * 2 <= kblocks / 4 && tiles * ks < 2 * num_sms()) ks *= 2;
  return ks;
}

}  // namespace

namespace {

// Muon gradients of 128 x 512 / 512 x 128 run the tensor-core Newton-Schulz
// kernel, which keeps every operand on chip and needs no scratch.
bool ns_on_chip(const LactArgs& a) {
  return a.update_rule == LACT_UPDATE_MUON && a.dk == kN5 && a.dv == kN5 &&
         a.dh == kNsCluster * kN5;
}

struct Sizes {
  bool ok;
  int Z, chunk;
  bool split;
  int64_t nW[3], nrows[3], ns_stride;
  size_t f32n, bfn, bytes;
};

Sizes lact_sizes(const LactArgs& a) {
  Sizes z;
  memset(&z, 0, sizeof(z));
  z.ok = a.dtype == TTT_BF16 && a.dk == a.dv && (a.dk == 64 || a.dk == 128 || a.dk == 256) &&
         a.dh % 128 == 0 && a.dh <= 1024;
  if (!z.ok) return z;
  const int dk = a.dk, dv = a.dv, dh = a.dh;
  z.Z = a.B * a.H;
  z.chunk = a.T > 0 ? (a.chunk < a.T ? a.chunk : a.T) : 1;
  z.split = a.update_rule == LACT_UPDATE_MUON;
  z.nW[0] = z.nW[1] = (int64_t)dh * dk;
  z.nW[2] = (int64_t)dv * dh;
  z.nrows[0] = z.nrows[1] = dh;
  z.nrows[2] = dv;
  const int s_max = dk < dh ? dk : dh;
  z.ns_stride = 2 * kNsCluster * (int64_t)s_max * s_max +
                kNsCluster * 2 * (int64_t)s_max * s_max + (int64_t)dh * dk + 64;
  for (int m = 0; m < 3; ++m) z.f32n += (size_t)z.Z * (2 * z.nW[m] + z.nrows[m]);
  // Newton-Schulz scratch: only the general-shape kernel needs it (the
  // tensor-core kernel for 128 x 512 gradients keeps everything on chip)
  if (z.split && !ns_on_chip(a)) z.f32n += (size_t)z.Z * 3 * z.ns_stride;
  if (a.momentum) z.f32n += (size_t)z.Z * (z.nW[0] + z.nW[1] + z.nW[2]);
  z.bfn = (size_t)z.Z * (2 * dh * dk + dv * dh) * (z.split ? 2 : 1);
  z.bfn += (size_t)z.Z * z.chunk * dh * 4 * (z.split ? 2 : 1);
  z.bytes = z.f32n * 4 + z.bfn * 2 + 4096;
  return z;
}

}  // namespace

size_t lact_scratch_bytes(const LactArgs& a) {
  Sizes z = lact_sizes(a);
  return z.ok ? z.bytes : 0;
}

// The library's own stream-ordered memory pool on the current device. Its
// release threshold keeps freed scratch mapped, so back-to-back calls reuse it
// instead of mapping it again after every synchronisation (the device's
// default pool, and with it the caller's, is left untouched).
cudaMemPool_t scratch_pool() {
  constexpr int kMaxDevices = 64;
  static cudaMemPool_t pools[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props;
    memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    uint64_t keep = UINT64_MAX;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    pools[dev] = pool;
  }
  return pools[dev];
}

namespace {
std::atomic<int> g_fail_allocs{0};
}  // namespace

void set_failing_allocs(int n) { g_fail_allocs.store(n < 0 ? 0 : n); }

cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t s) {
  *p = nullptr;
  // test hook: the next n allocations fail as if the device were out of memory
  int n = g_fail_allocs.load();
  while (n > 0 && !g_fail_allocs.compare_exchange_weak(n, n - 1)) {
  }
  if (n > 0) return cudaErrorMemoryAllocation;
  cudaMemPool_t pool = scratch_pool();
  const cudaError_t e = pool ? cudaMallocFromPoolAsync(p, bytes, pool, s) : cudaMallocAsync(p, bytes, s);
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

ttt_status lact_forward(const LactArgs& a, cudaStream_t s) {
  const Sizes z = lact_sizes(a);
  if (!z.ok) return TTT_ERR_UNSUPPORTED;
  void* base = nullptr;
  if (scratch_alloc(&base, z.bytes, s) != cudaSuccess) return TTT_ERR_ALLOC;
  ttt_status r = lact_run(a, s, base, z.bytes);
  if (cudaFreeAsync(base, s) != cudaSuccess && r == TTT_OK) r = TTT_ERR_CUDA;
  return r;
}

ttt_status lact_run(const LactArgs& a, cudaStream_t s, void* base, size_t bytes) {
  const Sizes zz = lact_sizes(a);
  if (!zz.ok) return TTT_ERR_UNSUPPORTED;
  if (!base || bytes < zz.bytes || (reinterpret_cast<uintptr_t>(base) & 255u)) return TTT_ERR_ARG;
  const int Z = zz.Z, dk = a.dk, dv = a.dv, dh = a.dh;
  const int chunk = zz.chunk;
  const bool split = zz.split;
  const int64_t* nW = zz.nW;
  const int64_t* nrows = zz.nrows;
  const int64_t ns_stride = zz.ns_stride;
  Scratch sc;
  {
    // masters, then the three gradients back to back (one buffer for the
    // context-parallel exchange), then the row norms
    float* f = static_cast<float*>(base);
    for (int m = 0; m < 3; ++m) {
      sc.Wm[m] = f;
      f += Z * nW[m];
    }
    for (int m = 0; m < 3; ++m) {
      sc.G[m] = f;
      f += Z * nW[m];
    }
    for (int m = 0; m < 3; ++m) {
      sc.rho[m] = f;
      f += Z * nrows[m];
    }
    const bool ns_scratch = split && !ns_on_chip(a);
    sc.ns = ns_scratch ? f : nullptr;
    if (ns_scratch) f += (size_t)Z * 3 * ns_stride;
    for (int m = 0; m < 3; ++m) {
      sc.M[m] = a.momentum ? f : nullptr;
      if (a.momentum) f += Z * nW[m];
    }
    uintptr_t up = (reinterpret_cast<uintptr_t>(f) + 255) & ~uintptr_t(255);
    __nv_bfloat16* b = reinterpret_cast<__nv_bfloat16*>(up);
    auto take = [&](size_t n) {
      __nv_bfloat16* r = b;
      b += (n + 127) / 128 * 128;
      return r;
    };
    for (int x = 0; x < (split ? 2 : 1); ++x) {
      sc.w13[x] = take((size_t)Z * 2 * dh * dk);
      sc.w2[x] = take((size_t)Z * dv * dh);
      sc.aq[x] = take((size_t)Z * chunk * dh);
      sc.ak[x] = take((size_t)Z * chunk * dh);
      sc.dh1[x] = take((size_t)Z * chunk * dh);
      sc.dh3[x] = take((size_t)Z * chunk * dh);
    }
    if (!split)
      sc.w13[1] = sc.w13[0], sc.w2[1] = sc.w2[0], sc.aq[1] = sc.ak[1] = sc.dh1[1] = sc.dh3[1] = nullptr;
  }
  sc.ns_stride = ns_stride;

  ttt_status result = TTT_OK;
  auto check = [&](cudaError_t e) {
    if (e != cudaSuccess && result == TTT_OK) result = TTT_ERR_CUDA;
    return e == cudaSuccess;
  };

  RowArgs ra;
  memset(&ra, 0, sizeof(ra));
  for (int m = 0; m < 3; ++m) {
    ra.Wm[m] = sc.Wm[m];
    ra.rho[m] = sc.rho[m];
    ra.G[m] = sc.G[m];
  }
  // row-kernel matrix order is (W1, W3, W2); LactArgs::w_sb is (W1, W2, W3)
  ra.win_sz[0] = a.w_sb[0];
  ra.win_sz[1] = a.w_sb[2];
  ra.win_sz[2] = a.w_sb[1];
  ra.Win[0] = a.W1;
  ra.Win[1] = a.W3;
  ra.Win[2] = a.W2;
  ra.w13_hi = sc.w13[0];
  ra.w13_lo = sc.w13[1];
  ra.w2_hi = sc.w2[0];
  ra.w2_lo = sc.w2[1];
  ra.Z = Z;
  ra.H = a.H;
  ra.dk = dk;
  ra.dv = dv;
  ra.dh = dh;
  ra.split = split;
  ra.status = a.status;
  // momentum: LactArgs order (W1, W2, W3) -> row order (W1, W3, W2)
  ra.momentum = a.momentum;
  ra.beta = a.beta;
  {
    const int order[3] = {0, 2, 1};
    for (int m = 0; m < 3; ++m) {
      ra.M[m] = sc.M[m];
      ra.Min[m] = a.momentum ? a.M0[order[m]] : nullptr;
      ra.min_sz[m] = a.momentum ? a.m0_sb[order[m]] : 0;
    }
  }
  const int row_warps = Z * (2 * dh + dv);
  const int row_blocks = (row_warps * 32 + 255) / 256;
  ra.prep = 1;
  lact_rows_kernel<<<row_blocks, 256, 0, s>>>(ra);
  check(cudaGetLastError());
  ra.prep = 0;

  NsArgs na;
  memset(&na, 0, sizeof(na));
  if (split) {
    for (int m = 0; m < 3; ++m) na.G[m] = sc.G[m];
    na.rows[0] = na.rows[1] = dh;
    na.cols[0] = na.cols[1] = dk;
    na.rows[2] = dv;
    na.cols[2] = dh;
    na.scratch = sc.ns;
    na.status = a.status;
    na.scratch_stride = ns_stride;
    na.a = 3.4445f;
    na.b = -4.7750f;
    na.c = 2.0315f;
    na.eps = 1e-7f;
    na.steps = 5;
  }

  // Gradients of 512 x 128 / 128 x 512 run the shared-memory-resident kernel.
  const bool ns_tc = ns_on_chip(a);
  if (ns_tc)
    check(cudaFuncSetAttribute(ns5_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(sizeof(Ns5Smem) + 1024)));
  const int* segW = split ? &kSegBsplit[0][0] : &kSegExact[0][0];
  const int nsegW = split ? 2 : 1;

  // Tensor maps do not depend on the chunk (token operands carry the chunk
  // start as a row offset); the chunk-length activation maps are built once
  // for full chunks and once more for a ragged last chunk.
  Operand W13, W13h, W2mn, W2k, Qk0, Kk0, Vk0, Kmn0, Vmn0;
  struct ActOps {
    Operand AQk, DH1mn, DH3mn, AKmn;
  } act_full, act_last;
  CUtensorMap gmaps[3];
  if (a.T > 0) {
    bool ok = true;
    ok &= buf_op(W13, sc.w13, Z, 2 * dh, 2 * dh, dk, 0, BN, split);
    ok &= buf_op(W13h, sc.w13, Z, 2 * dh, 2 * dh, dk, 0, 2 * gemm::kHid, split);
    ok &= buf_op(W2mn, sc.w2, Z, dv, dv, dh, 1, 64, split);
    // the Y tiles are only as wide as dv when dv <= 128 (no columns of zeros)
    ok &= buf_op(W2k, sc.w2, Z, dv, dv, dh, 0, dv <= 128 ? 128 : BN, split);
    ok &= tok_kmajor(Qk0, a.q, a, dk, 0, gemm::BM);
    ok &= tok_kmajor(Kk0, a.k, a, dk, 0, gemm::BM);
    ok &= tok_kmajor(Vk0, a.v, a, dv, 0, gemm::BM);
    ok &= tok_mnmajor(Kmn0, a.k, a, dk, 0);
    ok &= tok_mnmajor(Vmn0, a.v, a, dv, 0);
    auto acts = [&](ActOps& o, int rows) {
      return buf_op(o.AQk, sc.aq, Z, rows, chunk, dh, 0, gemm::BM, split) &&
             buf_op(o.DH1mn, sc.dh1, Z, rows, chunk, dh, 1, 64, split) &&
             buf_op(o.DH3mn, sc.dh3, Z, rows, chunk, dh, 1, 64, split) &&
             buf_op(o.AKmn, sc.ak, Z, rows, chunk, dh, 1, 64, split);
    };
    ok &= acts(act_full, chunk);
    const int last = a.T > 0 ? a.T - ((a.T - 1) / chunk) * chunk : chunk;
    ok &= last == chunk ? true : acts(act_last, last);
    if (last == chunk) act_last = act_full;
    ok &= grad_map(&gmaps[0], sc.G[0], Z, dh, dk);
    ok &= grad_map(&gmaps[1], sc.G[1], Z, dh, dk);
    ok &= grad_map(&gmaps[2], sc.G[2], Z, dv, dh);
    if (!ok) result = TTT_ERR_CUDA;
  }

  for (int s0 = 0; s0 < a.T && result == TTT_OK; s0 += chunk) {
    const int bc = (a.T - s0) < chunk ? (a.T - s0) : chunk;
    // operands of this chunk
    Operand Qk = Qk0, Kk = Kk0, Vk = Vk0, Kmn = Kmn0, Vmn = Vmn0;
    Qk.row0 = Kk.row0 = Vk.row0 = Kmn.row0 = Vmn.row0 = s0;
    const ActOps& act = bc == chunk ? act_full : act_last;
    const Operand &AQk = act.AQk, &DH1mn = act.DH1mn, &DH3mn = act.DH3mn, &AKmn = act.AKmn;
    bool okm = true;  // output maps built
    auto new_problem = [&](Params& P) -> Problem& {
      Problem& p = P.p[P.nprob++];
      memset(&p, 0, sizeof(p));
      p.nz = Z;
      p.ksplit = 1;
      p.tn = BN;
      return p;
    };
    auto add_aq = [&](Params& P) {  // Aq = silu(Q W1^T) * (Q W3^T)
      Problem& p = new_problem(P);
      p.a = Qk;
      p.b = W13;
      p.M = bc;
      p.N = 2 * dh;
      p.K = dk;
      segs(p, nsegW, reinterpret_cast<const int(*)[2]>(segW));
      p.epi = gemm::EPI_AQ;
      p.e = epi_base(a, s0, bc);
      // The apply path produces only the layer output, so Aq is stored as
      // plain bf16 even under Muon (the weights keep their hi / lo parts).
      p.e.nsplit = 1;
      p.e.optr[0] = sc.aq[0];
      p.e.orows = chunk;
      p.e.ocols = dh;
    };
    auto add_y = [&](Params& P) {  // Y = Aq W2^T -> output tokens
      Problem& p = new_problem(P);
      p.a = AQk;
      p.b = W2k;
      p.M = bc;
      p.N = dv;
      p.K = dh;
      if (split)
        segs(p, 2, kSegBsplit);  // Aq (bf16) x W2 hi + Aq x W2 lo
      else
        segs(p, 1, kSegExact);
      p.epi = gemm::EPI_Y;
      p.tn = dv <= 128 ? 128 : BN;
      p.pair = split && p.tn <= 128 ? 1 : 0;  // Aq loaded once for both W2 parts
      p.e = epi_base(a, s0, bc);
      p.e.orow0 = s0;
    };
    auto add_key = [&](Params& P) {  // [H1 | H3 | V W2] tiles -> Ak', dH1, dH3
      Problem& p = new_problem(P);
      p.a = Kk;
      p.b = W13h;
      p.a2 = Vk;
      p.b2 = W2mn;
      p.M = bc;
      p.N = 2 * dh;
      p.K = dk;  // = dv
      p.tn = 2 * gemm::kHid;
      segs(p, nsegW, reinterpret_cast<const int(*)[2]>(segW));
      p.nseg2 = nsegW;
      for (int i = 0; i < nsegW; ++i) {
        p.seg2_a[i] = segW[2 * i];
        p.seg2_b[i] = segW[2 * i + 1];
      }
      p.epi = gemm::EPI_HKG;
      p.pair = split ? 1 : 0;  // K (and V) loaded once for the hi and lo weight parts
      p.e = epi_base(a, s0, bc);
      p.e.nsplit = split ? 2 : 1;
      for (int x = 0; x < (split ? 2 : 1); ++x) {
        p.e.optr[3 * x + 0] = sc.ak[x];
        p.e.optr[3 * x + 1] = sc.dh1[x];
        p.e.optr[3 * x + 2] = sc.dh3[x];
      }
      p.e.orows = chunk;
      p.e.ocols = dh;
    };
    auto add_grads = [&](Params& P) {  // weight gradients (token reductions, split-K)
      const int kblocks = (bc + gemm::BK - 1) / gemm::BK;
      const int tiles = Z * (2 * ((dh + gemm::BM - 1) / gemm::BM) * ((dk + BN - 1) / BN) +
                             ((dv + gemm::BM - 1) / gemm::BM) * ((dh + BN - 1) / BN));
      const int ks = pick_ksplit(kblocks, tiles);
      for (int g = 0; g < 3; ++g) {
        Problem& p = new_problem(P);
        p.ksplit = ks;
        p.K = bc;
        p.epi = gemm::EPI_GRAD;
        if (g < 2) {
          p.a = g == 0 ? DH1mn : DH3mn;
          p.b = Kmn;
          p.M = dh;
          p.N = dk;
          p.tn = dk <= 128 ? 128 : BN;  // (MN-major B: loaded in 64-column boxes)
          if (split)
            segs(p, 2, kSegAsplit);
          else
            segs(p, 1, kSegExact);
          p.pair = split && p.tn <= 128 ? 2 : 0;  // K loaded once for the dH hi and lo parts
          p.e = epi_base(a, s0, dh);
          p.e.ozdiv = Z;
          p.e.gmap = gmaps[g];
        } else {
          p.a = Vmn;
          p.b = AKmn;
          p.M = dv;
          p.N = dh;
          if (split)
            segs(p, 2, kSegBsplit);
          else
            segs(p, 1, kSegExact);
          p.e = epi_base(a, s0, dv);
          p.e.ozdiv = Z;
          p.e.scale = -1.f;
          p.e.gmap = gmaps[2];
        }
      }
    };
    auto run = [&](Params& P) {
      if (!okm) result = TTT_ERR_CUDA;
      check(launch_gemm(P, s));
    };
    // L1: Aq (causal) and the fused key-side tiles
    {
      Params P;
      memset(&P, 0, sizeof(P));
      P.status = a.status;
      if (a.causal) add_aq(P);
      add_key(P);
      run(P);
    }
    // L2: Y (causal) and the weight gradients
    {
      Params P;
      memset(&P, 0, sizeof(P));
      P.status = a.status;
      if (a.causal) add_y(P);
      add_grads(P);
      run(P);
    }
    // context parallelism: sum the gradients over the ranks that hold the
    // other token shards of this chunk
    if (a.reduce && result == TTT_OK) {
      if (a.reduce(sc.G[0], (size_t)Z * (nW[0] + nW[1] + nW[2]), s, a.reduce_user) != 0)
        result = TTT_ERR_CUDA;
      if (result != TTT_OK) break;
    }
    // L3 / L4: Muon orthogonalisation, update and row renormalisation
    if (split) {
      if (ns_tc) {
        check(launch_pdl(ns5_kernel, dim3(Z * 3 * kNsCluster), dim3(kT5Threads),
                         sizeof(Ns5Smem) + 1024, s, na));
      } else {
        check(launch_pdl(ns_kernel, dim3(Z * 3 * kNsCluster), dim3(kNsThreads), 0, s, na));
      }
    }
    check(launch_pdl(lact_rows_kernel, dim3(row_blocks), dim3(256), 0, s, ra));
    if (!a.causal) {
      Params P;
      memset(&P, 0, sizeof(P));
      P.status = a.status;
      add_aq(P);
      run(P);
      Params P2;
      memset(&P2, 0, sizeof(P2));
      P2.status = a.status;
      add_y(P2);
      run(P2);
    }
  }

  float* finals[3] = {a.W1_final, a.W3_final, a.W2_final};
  for (int m = 0; m < 3 && result == TTT_OK; ++m) {
    if (!finals[m]) continue;
    check(launch_pdl(copy_kernel, dim3(148), dim3(256), 0, s, finals[m], (const float*)sc.Wm[m],
                     (int64_t)Z * nW[m]));
  }
  float* mfinals[3] = {a.M_final[0], a.M_final[2], a.M_final[1]};
  for (int m = 0; m < 3 && result == TTT_OK && a.momentum; ++m) {
    if (!mfinals[m]) continue;
    check(launch_pdl(copy_kernel, dim3(148), dim3(256), 0, s, mfinals[m], (const float*)sc.M[m],
                     (int64_t)Z * nW[m]));
  }
  return result;
}

}  // namespace ttt
