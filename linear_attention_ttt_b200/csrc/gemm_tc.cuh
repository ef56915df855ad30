// Grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA)
// with the fused epilogues of the LaCT chunk step.
//
// Each problem computes, per batch index z (a (batch, head) pair),
//     D_z[M x N] = sum_seg A_seg,z[M x K] * B_seg,z[N x K]^T
// over 1-3 "segments" (operand pairs accumulated into the same TMEM
// accumulator; used for split-precision products hi*hi + lo*hi + hi*lo).
// Operands are bf16 tensors read by TMA with the 128-byte swizzle, either
// K-major (storage [rows=M|N][K]) or MN-major (storage [rows=K][M|N]).
// Tiles are 128 x BN with a 64-wide K step. The kernel is persistent: each CTA
// walks the tile list (all problems of the launch) with stride gridDim.x.
// Warp roles: warp 0 issues TMA loads into a ring of kStages shared-memory
// stages; warp 1 owns two TMEM accumulators and one elected thread issues
// tcgen05.mma into them alternately; warps 2-9 run the epilogue of one
// accumulator (two warps per 32-lane quarter of TMEM, each taking half of the
// tile's columns) while the MMAs of the next tile fill the other. The epilogue
// writes through TMA: each warp stages 32 rows x 16 columns in shared memory
// and issues a tensor store (or an fp32 add-reduction for split-K gradients),
// so global writes are full row segments. All barrier waits are bounded.
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace ttt {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 320;   // 2 + 8 warps
constexpr int kEpiWarps = 8;
constexpr int kMaxProblems = 4;

enum Epi : int {
  EPI_GZ = 0,     // gz = -eta_i * D  (fp32, lane-interleaved layout, see gz_off)
  EPI_AQ = 1,     // aq = silu(h1) * h3                  (bf16 hi [+lo])
  EPI_HK = 2,     // ak = eta*silu(h1)*h3, dh3 = gz*silu(h1), dh1 = gz*h3*silu'(h1)
                  // (for both, a BN-wide tile holds BN/2 h1 columns, then the
                  //  BN/2 matching h3 columns)
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
  // TMA maps of the outputs, boxes of {16 columns, 32 rows, 1, 1}:
  //  EPI_AQ: omap[0] aq hi, [3] aq lo; EPI_HK: omap[0..2] ak, dh1, dh3 hi, [3..5] lo;
  //  EPI_Y: omap[0] output tokens {dv, T, H, B}; EPI_GRAD: omap[0] g {N, M, Z, 1}.
  CUtensorMap omap[6];
  int nsplit;              // 1 or 2 (bf16 outputs with residuals)
  int ozdiv;               // z -> (z % ozdiv, z / ozdiv) for output coords 2, 3
  int orow0;               // output row offset (chunk start for EPI_Y)
  float* gz;               // EPI_GZ destination / EPI_HK source
  int64_t gz_rows;         // rows per z of the gz layout (allocated chunk length)
  int gz_cols;             // hidden units
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
  alignas(128) float ostage[kEpiWarps][2][32 * 16];  // per-warp TMA store staging (x2)
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2];
  uint32_t tmem_base;
};

// Offset of gz element (z, row, col) in the lane-interleaved layout
// [z][col/16][row][16]: 32 consecutive rows x 16 columns are 2 KB contiguous,
// so a warp (one row per lane) reads or writes them fully coalesced.
__device__ __forceinline__ int64_t gz_off(const EpiArgs& e, int z, int row, int col) {
  return ((((int64_t)z * (e.gz_cols / 16) + col / 16) * e.gz_rows + row) << 4) + (col & 15);
}

// Per-warp TMA output staging: lane = tile row, 16 columns per store.
struct Stager {
  float* buf[2];
  int lane, next;

  __device__ __forceinline__ void* slot() {
    // the slot about to be rewritten was used two stores ago
    if (lane == 0) bulk_wait_read<1>();
    __syncwarp();
    return buf[next];
  }
  __device__ __forceinline__ void issue(const CUtensorMap* m, void* src, int c0, int c1, int c2,
                                        int c3, bool reduce) {
    umma::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (reduce)
        tma_reduce_add_4d(m, src, c0, c1, c2, c3);
      else
        tma_store_4d(m, src, c0, c1, c2, c3);
      bulk_commit();
    }
    next ^= 1;
  }
  __device__ __forceinline__ void f32(const CUtensorMap* m, const float (&v)[16], int c0, int c1,
                                      int c2, int c3, bool reduce) {
    float* d = static_cast<float*>(slot()) + lane * 16;
#pragma unroll
    for (int u = 0; u < 16; u += 4)
      *reinterpret_cast<float4*>(d + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
    issue(m, d - lane * 16, c0, c1, c2, c3, reduce);
  }
  // bf16 of v (lo = false) or of the residual v - bf16(v) (lo = true)
  __device__ __forceinline__ void bf16(const CUtensorMap* m, const float (&v)[16], bool lo, int c0,
                                       int c1, int c2, int c3) {
    __nv_bfloat16* d = static_cast<__nv_bfloat16*>(slot()) + lane * 16;
    __align__(16) __nv_bfloat16 o[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v[u]);
      o[u] = lo ? __float2bfloat16_rn(v[u] - __bfloat162float(h)) : h;
    }
    reinterpret_cast<uint4*>(d)[0] = reinterpret_cast<const uint4*>(o)[0];
    reinterpret_cast<uint4*>(d)[1] = reinterpret_cast<const uint4*>(o)[1];
    issue(m, d - lane * 16, c0, c1, c2, c3, false);
  }
};


struct TileCoord {
  int pi, z, ks, m0, n0;
};

__device__ __forceinline__ TileCoord decode_tile(const Params& P, int t) {
  TileCoord c;
  int pi = 0;
  while (pi + 1 < P.nprob && t >= P.p[pi + 1].tile_begin) ++pi;
  const Problem& pr = P.p[pi];
  int local = t - pr.tile_begin;
  const int nt = local % pr.ntiles;
  local /= pr.ntiles;
  const int mt = local % pr.mtiles;
  local /= pr.mtiles;
  c.pi = pi;
  c.ks = local % pr.ksplit;
  c.z = local / pr.ksplit;
  c.m0 = mt * BM;
  c.n0 = nt;  // n-tile index; the kernel scales it by BN
  return c;
}

__device__ __forceinline__ float sigmoidf_(float x) { return __frcp_rn(1.f + __expf(-x)); }

// Epilogue for 16 consecutive accumulator columns [c0, c0+16) of row `row` of
// tile (m0, n0). For EPI_AQ / EPI_HK the tile's 128 columns hold 64 columns of
// silu-branch pre-activations (h1) followed by the 64 matching h3 columns; the
// caller passes v1 = h1 values and v3 = h3 values for hidden units
// [n0/2 + c0, n0/2 + c0 + 16).
__device__ __forceinline__ float eta_of(const EpiArgs& e, int z, int row) {
  const int b = z / e.H, h = z % e.H;
  return e.eta.p[b * e.eta.sb + h * e.eta.sh + (int64_t)(e.eta_t0 + row) * e.eta.st];
}

// K-block range of one tile (one K split of it).
__device__ __forceinline__ void k_range(const Problem& pr, int ks, int& kb0, int& nk) {
  const int kblocks = (pr.K + BK - 1) / BK;
  const int kb_per = (kblocks + pr.ksplit - 1) / pr.ksplit;
  kb0 = ks * kb_per;
  nk = max(0, min(kblocks, kb0 + kb_per) - kb0);
}

// Epilogue of one accumulator tile, run by one warp: its 32 TMEM lanes (tile
// rows quarter*32 ...) and the columns of half `ch` (0 or 1) of the tile.
// Rows and columns outside an output tensor are clipped by TMA; rows between
// the chunk end and the tensor end may receive values that the caller's later
// work overwrites or never reads.
template <int BN>
__device__ __forceinline__ void epilogue_tile(const Problem& pr, const TileCoord& tc, int quarter,
                                              uint32_t tbase, bool live_tile, int ch, Stager& sg) {
  const EpiArgs& e = pr.e;
  const int z = tc.z, n0 = tc.n0 * BN;
  const int row0 = tc.m0 + quarter * 32;  // first tile row of this warp
  const int lim = min(pr.M, e.rows_valid);
  const bool live = live_tile && row0 < lim;    // warp-uniform
  const int grow = row0 + sg.lane;
  const bool lane_ok = grow < lim;              // this lane's row exists
  const int oz2 = z % e.ozdiv, oz3 = z / e.ozdiv;
  if (pr.epi == EPI_AQ || pr.epi == EPI_HK) {
    constexpr int HALF = BN / 2;
    const int hid0 = n0 / 2;  // first hidden unit of this tile
    float eta_i = 0.f;
    if (live && pr.epi == EPI_HK && lane_ok) eta_i = eta_of(e, z, grow);
    for (int c = ch * (HALF / 2); c < (ch + 1) * (HALF / 2); c += 16) {
      float h1[16], h3[16];
      umma::tmem_ld16(tbase + c, h1);
      umma::tmem_ld16(tbase + HALF + c, h3);
      if (!live) continue;
      const int col = hid0 + c;
      float sgm[16], s1[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        sgm[u] = sigmoidf_(h1[u]);
        s1[u] = h1[u] * sgm[u];
      }
      if (pr.epi == EPI_AQ) {
        float a[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) a[u] = s1[u] * h3[u];
        for (int x = 0; x < e.nsplit; ++x) sg.bf16(&e.omap[3 * x], a, x, col, row0, oz2, oz3);
      } else {
        float g[16] = {};
        if (lane_ok) {
          const float* gp = e.gz + gz_off(e, z, grow, col);
#pragma unroll
          for (int u = 0; u < 16; u += 4) {
            const float4 t = *reinterpret_cast<const float4*>(gp + u);
            g[u] = t.x, g[u + 1] = t.y, g[u + 2] = t.z, g[u + 3] = t.w;
          }
        }
        float ak[16], d3[16], d1[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          ak[u] = eta_i * s1[u] * h3[u];
          d3[u] = g[u] * s1[u];
          d1[u] = g[u] * h3[u] * sgm[u] * (1.f + h1[u] * (1.f - sgm[u]));
        }
        for (int x = 0; x < e.nsplit; ++x) {
          sg.bf16(&e.omap[3 * x + 0], ak, x, col, row0, oz2, oz3);
          sg.bf16(&e.omap[3 * x + 1], d1, x, col, row0, oz2, oz3);
          sg.bf16(&e.omap[3 * x + 2], d3, x, col, row0, oz2, oz3);
        }
      }
    }
    return;
  }
  float eta_i = 0.f;
  if (live && pr.epi == EPI_GZ && lane_ok) eta_i = eta_of(e, z, grow);
  for (int c = ch * (BN / 2); c < (ch + 1) * (BN / 2); c += 16) {
    float v[16];
    umma::tmem_ld16(tbase + c, v);
    const int gc = n0 + c;
    if (!live || gc >= pr.N) continue;
    if (pr.epi == EPI_GZ) {
      if (!lane_ok) continue;
      float* gp = e.gz + gz_off(e, z, grow, gc);
#pragma unroll
      for (int u = 0; u < 16; u += 4)
        *reinterpret_cast<float4*>(gp + u) =
            make_float4(-eta_i * v[u], -eta_i * v[u + 1], -eta_i * v[u + 2], -eta_i * v[u + 3]);
    } else if (pr.epi == EPI_GRAD) {
      if (e.scale != 1.f)
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] *= e.scale;
      sg.f32(&e.omap[0], v, gc, row0, oz2, oz3, true);
    } else {  // EPI_Y
      if (e.out_bf16)
        sg.bf16(&e.omap[0], v, false, gc, e.orow0 + row0, oz2, oz3);
      else
        sg.f32(&e.omap[0], v, gc, e.orow0 + row0, oz2, oz3, false);
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<BN>& sm = *reinterpret_cast<Smem<BN>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.acc_full[x], 1);
      mbar_init(&sm.acc_empty[x], kEpiWarps);
    }
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(&sm.tmem_base, 2 * BN);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer: one continuous ring over all tiles ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x) {
        const TileCoord tc = decode_tile(P, t);
        const Problem& pr = P.p[tc.pi];
        int kb0, nk;
        k_range(pr, tc.ks, kb0, nk);
        const Operand& A = pr.a;
        const Operand& B = pr.b;
        const int az2 = tc.z % A.zdiv, az3 = tc.z / A.zdiv, bz2 = tc.z % B.zdiv,
                  bz3 = tc.z / B.zdiv;
        const int m0 = tc.m0, n0 = tc.n0 * BN;
        for (int seg = 0; seg < pr.nseg && ok; ++seg) {
          const CUtensorMap* am = &A.map[pr.seg_a[seg]];
          const CUtensorMap* bm = &B.map[pr.seg_b[seg]];
          for (int kb = kb0; kb < kb0 + nk; ++kb, ++it) {
            const int st = it % kStages;
            if (it >= kStages && !mbar_wait(&sm.empty[st], ((it / kStages) - 1) & 1, P.status)) {
              ok = false;
              break;
            }
            const int k = kb * BK;
            mbar_arrive_expect_tx(&sm.full[st], (BM + BN) * BK * 2);
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
                tma_load_4d(sm.b[st] + x * 8192, bm, &sm.full[st], n0 + 64 * x, B.row0 + k, bz2,
                            bz3);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.total_tiles && ok; t += gridDim.x, ++lt) {
        const TileCoord tc = decode_tile(P, t);
        const Problem& pr = P.p[tc.pi];
        int kb0, nk;
        k_range(pr, tc.ks, kb0, nk);
        const int niter = nk * pr.nseg;
        const int ab = lt & 1;
        if (lt >= 2 && !mbar_wait(&sm.acc_empty[ab], ((lt >> 1) - 1) & 1, P.status)) break;
        umma::fence_after();
        const uint32_t dacc = tmem + ab * BN;
        const uint32_t idesc = umma::instr_desc(1, BM, BN, pr.a.mn_major, pr.b.mn_major);
        for (int i = 0; i < niter; ++i, ++it) {
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
            umma::mma_bf16(dacc, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma::commit(&sm.empty[st]);
        }
        umma::commit(&sm.acc_full[ab]);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9 ----------------
    const int quarter = warp & 3;
    const int ch = (warp - 2) >> 2;       // column half
    Stager sgr{{sm.ostage[warp - 2][0], sm.ostage[warp - 2][1]}, lane, 0};
    int lt = 0;
    for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++lt) {
      const TileCoord tc = decode_tile(P, t);
      const Problem& pr = P.p[tc.pi];
      int kb0, nk;
      k_range(pr, tc.ks, kb0, nk);
      const int ab = lt & 1;
      const bool waited = mbar_wait(&sm.acc_full[ab], (lt >> 1) & 1, P.status);
      umma::fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + ab * BN;
      epilogue_tile<BN>(pr, tc, quarter, tbase, waited && nk > 0, ch, sgr);
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
      if (!waited) break;
    }
    if (lane == 0) bulk_wait_all();  // every output write has landed
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, 2 * BN);
}

}  // namespace gemm
}  // namespace ttt
