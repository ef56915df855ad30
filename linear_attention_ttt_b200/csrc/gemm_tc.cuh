// Grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA)
// with the fused epilogues of the LaCT chunk step.
//
// Each problem computes, per batch index z (a (batch, head) pair),
//     D_z[M x N] = sum_seg A_seg,z[M x K] * B_seg,z[N x K]^T
// over 1-3 "segments" (operand pairs accumulated into the same TMEM
// accumulator; used for split-precision products hi*hi + lo*hi + hi*lo).
// Operands are bf16 tensors read by TMA with the 128-byte swizzle, either
// K-major (storage [rows=M|N][K]) or MN-major (storage [rows=K][M|N]).
// Tiles are 128 x BN with a 64-wide K step; one CTA computes one output tile
// (optionally one K-split of it). Warp roles: warp 0 issues TMA loads into a
// ring of kStages shared-memory stages, warp 1 owns the TMEM accumulator and
// one elected thread issues tcgen05.mma, warps 2-5 run the epilogue (each
// warp reads its 32-lane quarter of TMEM). All barrier waits are bounded.
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace ttt {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kMaxProblems = 4;

enum Epi : int {
  EPI_GZ = 0,     // gz[z][i][h] = -eta_i * D           (fp32)
  EPI_AQ = 1,     // aq = silu(h1) * h3                  (bf16 hi [+lo])
  EPI_HK = 2,     // ak = eta*silu(h1)*h3, dh3 = gz*silu(h1), dh1 = gz*h3*silu'(h1)
  EPI_Y = 3,      // out tokens = D                      (bf16 or fp32, strided)
  EPI_GRAD = 4,   // g[z][m][n] += scale * D             (fp32 atomics, split-K)
};

struct Operand {
  CUtensorMap map[2];  // [0] = hi / exact, [1] = lo residual (if used)
  int mn_major;        // 0: storage [rows = M|N][K]; 1: storage [rows = K][M|N]
  int row0;            // offset added to the storage-row coordinate
  int zdiv;            // z -> coords (z % zdiv, z / zdiv)
};

struct EpiArgs {
  float* f32;              // EPI_GZ / EPI_GRAD destination [z][rows][cols]
  int64_t f32_sz, f32_sr;
  __nv_bfloat16* bo[3];    // bf16 outputs [z][rows][cols]: hi parts
  __nv_bfloat16* bo_lo[3]; // lo residuals (null when not split)
  int64_t b_sz, b_sr;
  const float* gz;         // EPI_HK input [z][rows][cols]
  int64_t gz_sz, gz_sr;
  EtaView eta;             // per-token learning rates
  int eta_t0;              // chunk start (token index of row 0)
  int H;                   // heads (z = b * H + h)
  TokViewMut out;          // EPI_Y destination
  int out_bf16;
  int rows_valid;          // rows >= rows_valid are not written
  float scale;             // EPI_GRAD sign
};

struct Problem {
  Operand a, b;
  int M, N, K;      // K per segment
  int nseg;
  int seg_a[3], seg_b[3];
  int nz, ksplit, mtiles, ntiles, tile_begin;
  int epi;
  EpiArgs e;
};

struct Params {
  Problem p[kMaxProblems];
  int nprob;
  int total_tiles;
  int* status;
};

template <int BN>
struct Smem {
  alignas(1024) uint8_t a[kStages][BM * BK * 2];
  alignas(1024) uint8_t b[kStages][BN * BK * 2];
  uint64_t full[kStages], empty[kStages], accum;
  uint32_t tmem_base;
};

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }

__device__ __forceinline__ void store_split(__nv_bfloat16* hi, __nv_bfloat16* lo, int64_t off,
                                            const float* v, int n) {
  // n values (n % 8 == 0) -> bf16 hi (+ bf16 of the residual), 16-byte stores
  for (int j = 0; j < n; j += 8) {
    __align__(16) __nv_bfloat16 h[8], l[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      h[u] = __float2bfloat16_rn(v[j + u]);
      l[u] = __float2bfloat16_rn(v[j + u] - __bfloat162float(h[u]));
    }
    *reinterpret_cast<uint4*>(hi + off + j) = *reinterpret_cast<const uint4*>(h);
    if (lo) *reinterpret_cast<uint4*>(lo + off + j) = *reinterpret_cast<const uint4*>(l);
  }
}

// Epilogue for 16 consecutive accumulator columns [c0, c0+16) of row `row` of
// tile (m0, n0). For EPI_AQ / EPI_HK the tile's 128 columns hold 64 columns of
// silu-branch pre-activations (h1) followed by the 64 matching h3 columns; the
// caller passes v1 = h1 values and v3 = h3 values for hidden units
// [n0/2 + c0, n0/2 + c0 + 16).
__device__ __forceinline__ float eta_of(const EpiArgs& e, int z, int row) {
  const int b = z / e.H, h = z % e.H;
  return e.eta.p[b * e.eta.sb + h * e.eta.sh + (int64_t)(e.eta_t0 + row) * e.eta.st];
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<BN>& sm = *reinterpret_cast<Smem<BN>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile ----
  int pi = 0;
  while (pi + 1 < P.nprob && (int)blockIdx.x >= P.p[pi + 1].tile_begin) ++pi;
  const Problem& pr = P.p[pi];
  int local = blockIdx.x - pr.tile_begin;
  const int nt = local % pr.ntiles;
  local /= pr.ntiles;
  const int mt = local % pr.mtiles;
  local /= pr.mtiles;
  const int ks = local % pr.ksplit;
  const int z = local / pr.ksplit;
  const int m0 = mt * BM, n0 = nt * BN;
  const int kblocks = (pr.K + BK - 1) / BK;
  const int kb_per = (kblocks + pr.ksplit - 1) / pr.ksplit;
  const int kb0 = ks * kb_per, kb1 = min(kblocks, kb0 + kb_per);
  const int nk = max(0, kb1 - kb0);
  const int niter = nk * pr.nseg;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(&sm.tmem_base, BN);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0 && niter > 0) {
      const Operand& A = pr.a;
      const Operand& B = pr.b;
      const int az2 = z % A.zdiv, az3 = z / A.zdiv, bz2 = z % B.zdiv, bz3 = z / B.zdiv;
      const uint32_t bytes = (BM + BN) * BK * 2;
      for (int it = 0; it < niter; ++it) {
        const int st = it % kStages;
        if (it >= kStages && !mbar_wait(&sm.empty[st], ((it / kStages) - 1) & 1, P.status))
          break;
        const int seg = it / nk, kb = kb0 + it % nk;
        const CUtensorMap* am = &A.map[pr.seg_a[seg]];
        const CUtensorMap* bm = &B.map[pr.seg_b[seg]];
        const int k = kb * BK;
        mbar_arrive_expect_tx(&sm.full[st], bytes);
        if (!A.mn_major) {
          tma_load_4d(sm.a[st], am, &sm.full[st], k, A.row0 + m0, az2, az3);
        } else {
          tma_load_4d(sm.a[st], am, &sm.full[st], m0, A.row0 + k, az2, az3);
          tma_load_4d(sm.a[st] + 8192, am, &sm.full[st], m0 + 64, A.row0 + k, az2, az3);
        }
        if (!B.mn_major) {
          tma_load_4d(sm.b[st], bm, &sm.full[st], k, B.row0 + n0, bz2, bz3);
        } else {
#pragma unroll
          for (int x = 0; x < BN / 64; ++x)
            tma_load_4d(sm.b[st] + x * 8192, bm, &sm.full[st], n0 + 64 * x, B.row0 + k, bz2, bz3);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma::instr_desc(1, BM, BN, pr.a.mn_major, pr.b.mn_major);
      bool ok = true;
      for (int it = 0; it < niter && ok; ++it) {
        const int st = it % kStages;
        if (!mbar_wait(&sm.full[st], (it / kStages) & 1, P.status)) {
          ok = false;
          break;
        }
        umma::fence_after();
        const uint32_t sa = smem_u32(sm.a[st]), sb = smem_u32(sm.b[st]);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = pr.a.mn_major ? umma::smem_desc(sa + kk * 2048, 8192, 1024)
                                            : umma::smem_desc(sa + kk * 32, 16, 1024);
          const uint64_t bd = pr.b.mn_major ? umma::smem_desc(sb + kk * 2048, 8192, 1024)
                                            : umma::smem_desc(sb + kk * 32, 16, 1024);
          umma::mma_bf16(tmem, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma::commit(&sm.empty[st]);
      }
      umma::commit(&sm.accum);
    }
  } else {
    // ---------------- epilogue: warps 2..5 ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // tile row == TMEM lane
    const int grow = m0 + row;
    const bool waited = mbar_wait(&sm.accum, 0, P.status);
    umma::fence_after();
    const EpiArgs& e = pr.e;
    const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool live = waited && niter > 0 && grow < pr.M && grow < e.rows_valid;
    if (pr.epi == EPI_AQ || pr.epi == EPI_HK) {
      const int hid0 = n0 / 2;  // first hidden unit of this tile
      float eta_i = 0.f;
      if (live && pr.epi == EPI_HK) eta_i = eta_of(e, z, grow);
      for (int c = 0; c < 64; c += 16) {
        float h1[16], h3[16];
        umma::tmem_ld16(tbase + c, h1);
        umma::tmem_ld16(tbase + 64 + c, h3);
        if (!live) continue;
        const int64_t off = z * e.b_sz + (int64_t)grow * e.b_sr + hid0 + c;
        float s1[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) s1[u] = h1[u] * sigmoidf_(h1[u]);
        if (pr.epi == EPI_AQ) {
          float a[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) a[u] = s1[u] * h3[u];
          store_split(e.bo[0], e.bo_lo[0], off, a, 16);
        } else {
          const float* gzr = e.gz + z * e.gz_sz + (int64_t)grow * e.gz_sr + hid0 + c;
          float ak[16], d3[16], d1[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float g = gzr[u];
            const float sg = sigmoidf_(h1[u]);
            ak[u] = eta_i * s1[u] * h3[u];
            d3[u] = g * s1[u];
            d1[u] = g * h3[u] * sg * (1.f + h1[u] * (1.f - sg));
          }
          store_split(e.bo[0], e.bo_lo[0], off, ak, 16);
          store_split(e.bo[1], e.bo_lo[1], off, d1, 16);
          store_split(e.bo[2], e.bo_lo[2], off, d3, 16);
        }
      }
    } else {
      float eta_i = 0.f;
      if (live && pr.epi == EPI_GZ) eta_i = eta_of(e, z, grow);
      for (int c = 0; c < BN; c += 16) {
        float v[16];
        umma::tmem_ld16(tbase + c, v);
        if (!live) continue;
        const int gc = n0 + c;
        if (gc >= pr.N) continue;
        if (pr.epi == EPI_GZ) {
          float* d = e.f32 + z * e.f32_sz + (int64_t)grow * e.f32_sr + gc;
#pragma unroll
          for (int u = 0; u < 16; u += 4)
            *reinterpret_cast<float4*>(d + u) =
                make_float4(-eta_i * v[u], -eta_i * v[u + 1], -eta_i * v[u + 2], -eta_i * v[u + 3]);
        } else if (pr.epi == EPI_GRAD) {
          float* d = e.f32 + z * e.f32_sz + (int64_t)grow * e.f32_sr + gc;
#pragma unroll
          for (int u = 0; u < 16; ++u) atomicAdd(d + u, e.scale * v[u]);
        } else {  // EPI_Y
          const int b = z / e.H, h = z % e.H;
          const int64_t off = b * e.out.sb + h * e.out.sh + (int64_t)(e.eta_t0 + grow) * e.out.st + gc;
          if (e.out_bf16) {
            __align__(16) __nv_bfloat16 o[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) o[u] = __float2bfloat16_rn(v[u]);
            __nv_bfloat16* d = static_cast<__nv_bfloat16*>(e.out.p) + off;
            reinterpret_cast<uint4*>(d)[0] = reinterpret_cast<const uint4*>(o)[0];
            reinterpret_cast<uint4*>(d)[1] = reinterpret_cast<const uint4*>(o)[1];
          } else {
            float* d = static_cast<float*>(e.out.p) + off;
#pragma unroll
            for (int u = 0; u < 16; u += 4)
              *reinterpret_cast<float4*>(d + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
          }
        }
      }
    }
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, BN);
}

}  // namespace gemm
}  // namespace ttt
