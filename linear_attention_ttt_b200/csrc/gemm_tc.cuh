// Grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA)
// with the fused epilogues of the LaCT chunk step.
//
// Each problem computes, per batch index z (a (batch, head) pair),
//     D_z[M x N] = sum_seg A_seg,z[M x K] * B_seg,z[N x K]^T
// over 1-3 "segments" (operand pairs accumulated into the same TMEM
// accumulator; used for split-precision products hi*hi + lo*hi + hi*lo).
// A problem may carry a second product (operands a2, b2) whose tn/2 columns
// land beside the first product's tn columns in the same accumulator tile;
// the fused key-side LaCT epilogue uses it for V W2 next to K [W1; W3]^T.
// Operands are bf16 tensors read by TMA with the 128-byte swizzle, either
// K-major (storage [rows=M|N][K]) or MN-major (storage [rows=K][M|N]).
// Tiles are 128 x BN with a 64-wide K step. The kernel is persistent: each CTA
// walks the tile list (all problems of the launch) with stride gridDim.x.
// Warp roles: warp 0 issues TMA loads into a ring of kStages shared-memory
// stages; warp 1 owns two TMEM accumulators and one elected thread issues
// tcgen05.mma into them alternately; warps 2-9 run the epilogue of one
// accumulator (two warps per 32-lane quarter of TMEM, each taking half of the
// tile's columns) while the MMAs of the next tile fill the other. Each
// epilogue warp stages 32 rows x 128 bytes (64 bf16 or 32 fp32 columns) in its
// 128-byte-swizzled shared-memory buffer (conflict-free in both directions)
// and then writes it as full 128-byte row segments, four rows per store
// instruction; split-K gradients leave the same buffer as fp32 TMA
// add-reductions. All barrier waits are bounded.
#pragma once

#include <type_traits>

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

// W1 and W3 rows are interleaved in blocks of kHid (W13 rows: W1 0..63,
// W3 0..63, W1 64..127, ...), so a 2*kHid-wide column range of K W13^T holds
// h1 and h3 of the same kHid hidden units.
constexpr int kHid = 64;

enum Epi : int {
  EPI_AQ = 1,     // aq = silu(h1) * h3                  (bf16 hi [+lo])
  EPI_HKG = 2,    // tile [h1 | h3 | u] for kHid hidden units, u = (V W2) columns,
                  // gz = -eta_i u:  ak = eta*silu(h1)*h3, dh3 = gz*silu(h1),
                  // dh1 = gz*h3*silu'(h1)                 (bf16 hi [+lo])
  EPI_Y = 3,      // out tokens = D                      (bf16 or fp32, strided)
  EPI_GRAD = 4,   // g[z][m][n] += scale * D             (fp32 TMA add, split-K)
};

struct Operand {
  CUtensorMap map[2];  // [0] = hi / exact, [1] = lo residual (if used)
  int mn_major;        // 0: storage [rows = M|N][K]; 1: storage [rows = K][M|N]
  int row0;            // offset added to the storage-row coordinate
  int zdiv;            // z -> coords (z % zdiv, z / zdiv)
};

struct EpiArgs {
  // EPI_GRAD: TMA map of g {N, M, Z, 1} fp32, box {32, 32, 1, 1}, 128-byte swizzle.
  CUtensorMap gmap;
  // bf16 activation outputs [Z][orows][ocols] (row-major):
  //  EPI_AQ: optr[0] aq hi, [3] aq lo; EPI_HKG: optr[0..2] ak, dh1, dh3 hi, [3..5] lo.
  void* optr[6];
  int64_t orows;
  int ocols;
  int nsplit;              // 1 or 2 (bf16 outputs with residuals)
  int ozdiv;               // EPI_GRAD: z -> (z % ozdiv, z / ozdiv) for map coords 2, 3
  int orow0;               // output row offset (chunk start for EPI_Y)
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
  Operand a2, b2;   // second product (nseg2 > 0): tn/2 columns at accumulator column tn
  int M, N, K;      // K per segment (both products)
  int tn;           // tile width in columns of the first product (<= BN)
  int nseg, nseg2;
  // 0: one ring stage per segment and K block. 1: the two segments of each
  // product share A (maps seg_a[0] = seg_a[1]; B maps hi, lo): one stage holds
  // A, B0 and B1 (B1 at b + bn*BK*2). 2: they share B (A maps hi, lo): one
  // stage holds A0, B and A1 (A1 at b + bn*BK*2). Pairs need bn <= 128.
  int pair;
  int seg_a[3], seg_b[3], seg2_a[3], seg2_b[3];
  int nz, ksplit, mtiles, ntiles, tile_begin;
  // filled by fill_problem_tiles on the host: K blocks in total and per split,
  // and reciprocal multipliers ceil(2^32 / d) of ntiles, mtiles and ksplit, so
  // that the single-thread roles decode tiles without integer division
  int kblocks, kb_per;
  uint64_t mag_n, mag_m, mag_k;
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
  alignas(1024) uint8_t ostage[kEpiWarps][32 * 128];  // per-warp staging, swizzled
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2];
  uint32_t tmem_base;
};

// Per-warp staging buffers of 32 rows x 128 bytes with the 128-byte swizzle:
// 16-byte chunk j of row r sits at r * 128 + ((j ^ (r & 7)) << 4), so a lane
// writing its own row and eight lanes reading one row both hit 32 distinct
// banks per 128 bytes.
__device__ __forceinline__ uint32_t sw128(int r, int j) {
  return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// bf16 hi / lo parts of (a, b) as two packed words: hi = bf16(x) (round to
// nearest even), lo = bf16(x - hi). One paired conversion per part: a bf16 is
// the upper half of the float with the same value, so the float value of each
// hi half is recovered from the packed word by a shift or a mask. Equal to
// converting hi and lo element by element, with half the conversions.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a, b);
  lo = pack_bf16x2(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

// Row `lane` of the buffer, columns [16p, 16p + 16) as bf16 (chunks 2p, 2p+1):
// bf16(v), or the residual v - bf16(v) for LO.
template <bool LO>
__device__ __forceinline__ void put_bf16(uint8_t* s, int lane, int p, const float (&v)[16]) {
  uint32_t w[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    float a = v[2 * u], b = v[2 * u + 1];
    if constexpr (LO) {
      a -= __bfloat162float(__float2bfloat16_rn(a));
      b -= __bfloat162float(__float2bfloat16_rn(b));
    }
    w[u] = pack_bf16x2(a, b);
  }
  *reinterpret_cast<uint4*>(s + sw128(lane, 2 * p)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(s + sw128(lane, 2 * p + 1)) = make_uint4(w[4], w[5], w[6], w[7]);
}
// Row `lane`, fp32 columns [16p, 16p + 16) (chunks 4p .. 4p+3).
__device__ __forceinline__ void put_f32(uint8_t* s, int lane, int p, const float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<float4*>(s + sw128(lane, 4 * p + q)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
__device__ __forceinline__ void get_f32(const uint8_t* s, int lane, int p, float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 t = *reinterpret_cast<const float4*>(s + sw128(lane, 4 * p + q));
    v[4 * q] = t.x, v[4 * q + 1] = t.y, v[4 * q + 2] = t.z, v[4 * q + 3] = t.w;
  }
}
// Staged rows r < nrows -> dst + r * ld (bytes): each store instruction
// writes four complete 128-byte rows.
__device__ __forceinline__ void flush_rows(const uint8_t* s, int lane, uint8_t* dst, int64_t ld,
                                           int nrows) {
  __syncwarp();
  uint4 x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = *reinterpret_cast<const uint4*>(s + sw128(4 * i + (lane >> 3), lane & 7));
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + (lane >> 3);
    if (r < nrows) *reinterpret_cast<uint4*>(dst + r * ld + (lane & 7) * 16) = x[i];
  }
  __syncwarp();
}
// Rows r < nrows of src + r * ld (128 bytes each) -> staging (zeros beyond).
__device__ __forceinline__ void fill_rows(uint8_t* s, int lane, const uint8_t* src, int64_t ld,
                                          int nrows) {
  __syncwarp();
  uint4 x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + (lane >> 3);
    x[i] = r < nrows ? *reinterpret_cast<const uint4*>(src + r * ld + (lane & 7) * 16)
                     : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) *reinterpret_cast<uint4*>(s + sw128(4 * i + (lane >> 3), lane & 7)) = x[i];
  __syncwarp();
}

// Half-width staging: 32 rows x 64 bytes (2 KB), 16-byte chunk j (0..3) of row
// r at r * 64 + ((j ^ ((r >> 1) & 3)) << 4) -- conflict-free for a lane writing
// its row and for four lanes reading one row.
__device__ __forceinline__ uint32_t sw64(int r, int j) {
  return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}
template <bool LO>
__device__ __forceinline__ void put_bf16_64(uint8_t* s, int lane, int p, const float (&v)[16]) {
  uint32_t w[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    float a = v[2 * u], b = v[2 * u + 1];
    if constexpr (LO) {
      a -= __bfloat162float(__float2bfloat16_rn(a));
      b -= __bfloat162float(__float2bfloat16_rn(b));
    }
    w[u] = pack_bf16x2(a, b);
  }
  *reinterpret_cast<uint4*>(s + sw64(lane, 2 * p)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(s + sw64(lane, 2 * p + 1)) = make_uint4(w[4], w[5], w[6], w[7]);
}
// put_bf16_64<false> into sh and put_bf16_64<true> into sl, one conversion per part.
__device__ __forceinline__ void put_split_64(uint8_t* sh, uint8_t* sl, int lane, int p,
                                             const float (&v)[16]) {
  uint32_t h[8], l[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) split_bf16x2(v[2 * u], v[2 * u + 1], h[u], l[u]);
  *reinterpret_cast<uint4*>(sh + sw64(lane, 2 * p)) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(sh + sw64(lane, 2 * p + 1)) = make_uint4(h[4], h[5], h[6], h[7]);
  *reinterpret_cast<uint4*>(sl + sw64(lane, 2 * p)) = make_uint4(l[0], l[1], l[2], l[3]);
  *reinterpret_cast<uint4*>(sl + sw64(lane, 2 * p + 1)) = make_uint4(l[4], l[5], l[6], l[7]);
}
// Staged rows r < nrows (64 bytes each) -> dst + r * ld: eight rows per store.
__device__ __forceinline__ void flush_rows64(const uint8_t* s, int lane, uint8_t* dst, int64_t ld,
                                             int nrows) {
  __syncwarp();
  uint4 x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const uint4*>(s + sw64(8 * i + (lane >> 2), lane & 3));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 8 * i + (lane >> 2);
    if (r < nrows) *reinterpret_cast<uint4*>(dst + r * ld + (lane & 3) * 16) = x[i];
  }
  __syncwarp();
}

// The staging buffer of one epilogue warp. Synchronous use (stage, then
// flush_rows) needs no bookkeeping; a TMA add-reduction reads the buffer
// asynchronously, so the buffer is rewritten only after that read is done.
struct Stage {
  uint8_t* buf;
  int lane;
  bool pending;  // a TMA read may still be in flight (warp-uniform)
  int* status;   // device status word (index checks of the debug-bounds build)

  __device__ __forceinline__ void drain() {
    if (pending) {
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      pending = false;
    }
  }
  __device__ __forceinline__ void reduce(const CUtensorMap* m, int c0, int c1, int c2, int c3) {
    umma::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_reduce_add_4d(m, buf, c0, c1, c2, c3);
      bulk_commit();
    }
    pending = true;
  }
};

// Two 16-column TMEM loads in flight, then one wait.
__device__ __forceinline__ void tmem_ld2x16(uint32_t ta, uint32_t tb, float (&a)[16],
                                            float (&b)[16]) {
  uint32_t ra[16], rb[16];
  umma::tmem_ld16_async(ta, ra);
  umma::tmem_ld16_async(tb, rb);
  umma::tmem_wait_ld(ra);
  umma::tmem_wait_ld(rb);
#pragma unroll
  for (int u = 0; u < 16; ++u) a[u] = __uint_as_float(ra[u]), b[u] = __uint_as_float(rb[u]);
}


struct TileCoord {
  int pi, z, ks, m0, n0;
};

// floor(n / d) from mag = ceil(2^32 / d); exact for n * d < 2^32 (tile
// indices and counts here are far below 2^16).
__device__ __forceinline__ int div_mag(int n, uint64_t mag) {
  return (int)(((uint64_t)(uint32_t)n * mag) >> 32);
}

__device__ __forceinline__ TileCoord decode_tile(const Params& P, int t) {
  TileCoord c;
  int pi = 0;
  while (pi + 1 < P.nprob && t >= P.p[pi + 1].tile_begin) ++pi;
  const Problem& pr = P.p[pi];
  const int local = t - pr.tile_begin;
  const int q1 = div_mag(local, pr.mag_n);
  const int q2 = div_mag(q1, pr.mag_m);
  const int z = div_mag(q2, pr.mag_k);
  c.pi = pi;
  c.z = z;
  c.ks = q2 - z * pr.ksplit;
  c.m0 = (q1 - q2 * pr.mtiles) * BM;
  c.n0 = local - q1 * pr.ntiles;  // n-tile index; the kernel scales it by the problem's tile width
  return c;
}

// Logistic function from the fast exponential and the approximate division
// (relative error ~1e-7; 1 / inf = 0 for very negative x). A correctly rounded
// reciprocal costs about ten times as much and dominated the epilogues.
__device__ __forceinline__ float sigmoidf_(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// One special-function op instead of two: sigmoid(x) = (1 + tanh(x / 2)) / 2
// with the hardware tanh approximation (absolute error about 2.5e-4 on the
// result), used where the outputs are rounded to bf16 anyway.
__device__ __forceinline__ float sigmoid_fast(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
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

// K-block range of one tile (one K split of it).
__device__ __forceinline__ void k_range(const Problem& pr, int ks, int& kb0, int& nk) {
  kb0 = ks * pr.kb_per;
  nk = max(0, min(pr.kblocks, kb0 + pr.kb_per) - kb0);
}

// Epilogue of one accumulator tile, run by one warp: its 32 TMEM lanes (tile
// rows quarter*32 ...) and the columns of half `ch` (0 or 1) of the tile.
// Rows at or beyond min(M, rows_valid) are not written.
template <int BN, int EPI, bool SPLIT>
__device__ __forceinline__ void epilogue_body(const Problem& pr, const TileCoord& tc, int quarter,
                                              uint32_t tbase, int ch, Stage& sg) {
  const EpiArgs& e = pr.e;
  const int z = tc.z, n0 = tc.n0 * pr.tn;
  const int row0 = tc.m0 + quarter * 32;  // first tile row of this warp
  const int nrows = min(32, min(pr.M, e.rows_valid) - row0);
  const int lane = sg.lane;
  const bool lane_ok = lane < nrows;       // this lane's row exists
  uint8_t* const buf = sg.buf;
  sg.drain();
  if (!TTT_BOUNDS(z >= 0 && z < pr.nz && row0 >= 0 && row0 < pr.M && nrows <= 32, sg.status))
    return;
  // 64 bf16 columns of this warp's rows: values of columns [16p, 16p + 16)
  // from val(p, v), staged as bf16 (or as residuals for LO), then written.
  auto emit = [&](uint8_t* d, int64_t ld, auto lo_c, auto&& val) {
    constexpr bool LO = decltype(lo_c)::value;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float v[16];
      val(p, v);
      put_bf16<LO>(buf, lane, p, v);
    }
    flush_rows(buf, lane, d, ld, nrows);
  };
  using Hi = std::false_type;
  using Lo = std::true_type;

  if constexpr (EPI == EPI_AQ) {
    // tile columns [128ch, 128ch + 64) h1, [128ch + 64, 128ch + 128) h3
    const int64_t ld = (int64_t)e.ocols * 2;
    const int c0 = ch * 2 * kHid;
    const int hid = n0 / 2 + ch * kHid;
    if (!TTT_BOUNDS(hid + kHid <= e.ocols && row0 + nrows <= e.orows && c0 + 2 * kHid <= BN,
                    sg.status))
      return;
    auto aq = [&](int p, float (&a)[16]) {
      float h1[16], h3[16];
      tmem_ld2x16(tbase + c0 + 16 * p, tbase + c0 + kHid + 16 * p, h1, h3);
#pragma unroll
      for (int u = 0; u < 16; ++u)
        a[u] = h1[u] * (SPLIT ? sigmoidf_(h1[u]) : sigmoid_fast(h1[u])) * h3[u];
    };
    const int64_t off = (((int64_t)z * e.orows + row0) * e.ocols + hid) * 2;
    if constexpr (!SPLIT) {
      // four 16-column steps; the TMEM reads of the next step are issued right
      // after the wait for the current one and overlap its arithmetic
      uint32_t rb[2][2][16];
      auto issue = [&](int p) {
        umma::tmem_ld16_async(tbase + c0 + 16 * p, rb[p & 1][0]);
        umma::tmem_ld16_async(tbase + c0 + kHid + 16 * p, rb[p & 1][1]);
      };
      issue(0);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        umma::tmem_wait_ld(rb[p & 1][0]);
        umma::tmem_wait_ld(rb[p & 1][1]);
        if (p + 1 < 4) issue(p + 1);
        float a[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float h1 = __uint_as_float(rb[p & 1][0][u]), h3 = __uint_as_float(rb[p & 1][1][u]);
          a[u] = h1 * sigmoid_fast(h1) * h3;
        }
        put_bf16<false>(buf, lane, p, a);
      }
      flush_rows(buf, lane, static_cast<uint8_t*>(e.optr[0]) + off, ld, nrows);
    } else {
      emit(static_cast<uint8_t*>(e.optr[0]) + off, ld, Hi{}, aq);
      emit(static_cast<uint8_t*>(e.optr[3]) + off, ld, Lo{}, aq);
    }
  } else if constexpr (EPI == EPI_HKG) {
    // columns [0, 64) h1, [64, 128) h3, [128, 192) u of hidden units
    // hid .. hid + 63; this warp takes units [32ch, 32ch + 32). The sigmoid of
    // each h1 is evaluated once and kept; outputs go through the two 2 KB
    // halves of the staging buffer as 64-byte rows.
    const int64_t ld = (int64_t)e.ocols * 2;
    const int cw = ch * 32;
    const int hid = tc.n0 * kHid + cw;
    if (!TTT_BOUNDS(hid + 32 <= e.ocols && row0 + nrows <= e.orows && 2 * kHid + cw + 32 <= BN,
                    sg.status))
      return;
    const float eta_i = lane_ok ? eta_of(e, z, row0 + lane) : 0.f;
    auto dst = [&](int o) {
      return static_cast<uint8_t*>(e.optr[o]) + (((int64_t)z * e.orows + row0) * e.ocols + hid) * 2;
    };
    uint8_t* const bA = buf;
    uint8_t* const bB = buf + 2048;
    // Passes over the warp's 32 units in two 16-column steps each: ak (and, not
    // split, dh3), then dh3 (split), then dh1. Each step reads h1, h3 and u
    // from TMEM; the reads of the next step are issued right after the wait
    // for the current one, so their latency overlaps this step's arithmetic
    // (a wait covers every read of the thread issued before it).
    constexpr int kSteps = SPLIT ? 6 : 4;
    uint32_t rb[2][3][16];
    auto issue = [&](int st) {
      const int p = st & 1;
      umma::tmem_ld16_async(tbase + cw + 16 * p, rb[st & 1][0]);
      umma::tmem_ld16_async(tbase + kHid + cw + 16 * p, rb[st & 1][1]);
      umma::tmem_ld16_async(tbase + 2 * kHid + cw + 16 * p, rb[st & 1][2]);
    };
    float sgm[2][16];
    issue(0);
#pragma unroll
    for (int st = 0; st < kSteps; ++st) {
      const int p = st & 1;
      const int pass = SPLIT ? (st >> 1) : 2 * (st >> 1);  // 0: ak (+dh3), 1: dh3, 2: dh1
      umma::tmem_wait_ld(rb[st & 1][0]);
      umma::tmem_wait_ld(rb[st & 1][1]);
      umma::tmem_wait_ld(rb[st & 1][2]);
      if (st + 1 < kSteps) issue(st + 1);
      float h1[16], h3[16], gz[16], d[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        h1[u] = __uint_as_float(rb[st & 1][0][u]);
        h3[u] = __uint_as_float(rb[st & 1][1][u]);
        gz[u] = -eta_i * __uint_as_float(rb[st & 1][2][u]);
      }
      if (pass == 0) {
        float a[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          sgm[p][u] = SPLIT ? sigmoidf_(h1[u]) : sigmoid_fast(h1[u]);
          const float s1 = h1[u] * sgm[p][u];
          a[u] = eta_i * s1 * h3[u];
          d[u] = gz[u] * s1;
        }
        if constexpr (SPLIT) {
          put_split_64(bA, bB, lane, p, a);
        } else {
          put_bf16_64<false>(bA, lane, p, a);
          put_bf16_64<false>(bB, lane, p, d);
        }
      } else if (pass == 1) {
#pragma unroll
        for (int u = 0; u < 16; ++u) d[u] = gz[u] * h1[u] * sgm[p][u];
        put_split_64(bA, bB, lane, p, d);
      } else {
        // dh1 = gz h3 silu'(h1),  silu'(x) = sigmoid(x) (1 + x (1 - sigmoid(x)))
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float sg1 = sgm[p][u];
          d[u] = gz[u] * h3[u] * sg1 * (1.f + h1[u] * (1.f - sg1));
        }
        if constexpr (SPLIT)
          put_split_64(bA, bB, lane, p, d);
        else
          put_bf16_64<false>(bA, lane, p, d);
      }
      if (p == 1) {  // the pass's 32 units are staged
        if (pass == 0) {
          flush_rows64(bA, lane, dst(0), ld, nrows);
          flush_rows64(bB, lane, dst(SPLIT ? 3 : 2), ld, nrows);
        } else if (pass == 1) {
          flush_rows64(bA, lane, dst(2), ld, nrows);
          flush_rows64(bB, lane, dst(5), ld, nrows);
        } else {
          flush_rows64(bA, lane, dst(1), ld, nrows);
          if constexpr (SPLIT) flush_rows64(bB, lane, dst(4), ld, nrows);
        }
      }
    }
  } else if constexpr (EPI == EPI_GRAD) {
    const int oz2 = z % e.ozdiv, oz3 = z / e.ozdiv;
    for (int gi = 0; gi < pr.tn / 64; ++gi) {   // 32 fp32 columns per group
      const int gc = n0 + ch * (pr.tn / 2) + 32 * gi;
      if (gc >= pr.N) break;
      if (!TTT_BOUNDS((gc & 3) == 0 && gc - n0 + 32 <= BN, sg.status)) break;
      float v[16], w[16];
      tmem_ld2x16(tbase + gc - n0, tbase + gc - n0 + 16, v, w);
      const float sc = e.scale;
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] *= sc, w[u] *= sc;
      sg.drain();  // the previous reduction has read the buffer
      put_f32(buf, lane, 0, v);
      put_f32(buf, lane, 1, w);
      sg.reduce(&e.gmap, gc, row0, oz2, oz3);
    }
  } else {  // EPI_Y
    const int b = z / e.H, h = z % e.H;
    constexpr int64_t es = SPLIT ? 4 : 2;  // SPLIT selects fp32 output tokens here
    uint8_t* base = static_cast<uint8_t*>(e.out.p) +
                    ((int64_t)b * e.out.sb + (int64_t)h * e.out.sh +
                     (int64_t)(e.orow0 + row0) * e.out.st) * es;
    const int64_t ld = e.out.st * es;
    if constexpr (SPLIT) {
      // fp32 output tokens: 32 columns per group
      for (int gi = 0; gi < pr.tn / 64; ++gi) {
        const int gc = n0 + ch * (pr.tn / 2) + 32 * gi;
        if (gc >= pr.N) break;
        if (!TTT_BOUNDS(gc + 32 <= pr.N && gc - n0 + 32 <= BN, sg.status)) break;
        float v[16], w[16];
        tmem_ld2x16(tbase + gc - n0, tbase + gc - n0 + 16, v, w);
        put_f32(buf, lane, 0, v);
        put_f32(buf, lane, 1, w);
        flush_rows(buf, lane, base + (int64_t)gc * 4, ld, nrows);
      }
    } else {
      // bf16 output tokens: 64 columns per group
      for (int gi = 0; gi < pr.tn / 128; ++gi) {
        const int gc = n0 + ch * (pr.tn / 2) + 64 * gi;
        if (gc >= pr.N) break;
        if (!TTT_BOUNDS(gc + 64 <= pr.N && gc - n0 + 64 <= BN, sg.status)) break;
        auto y = [&](int p, float (&v)[16]) {
          uint32_t r[16];
          umma::tmem_ld16_async(tbase + gc - n0 + 16 * p, r);
          umma::tmem_wait_ld(r);
#pragma unroll
          for (int u = 0; u < 16; ++u) v[u] = __uint_as_float(r[u]);
        };
        emit(base + (int64_t)gc * 2, ld, Hi{}, y);
      }
    }
  }
}

// Epilogue of one accumulator tile, run by one warp: its 32 TMEM lanes (tile
// rows quarter*32 ...) and the columns of half `ch` (0 or 1) of the tile.
// Rows at or beyond min(M, rows_valid) are not written. Each (kind, precision)
// pair is a separate straight-line instantiation.
template <int BN>
__device__ __forceinline__ void epilogue_tile(const Problem& pr, const TileCoord& tc, int quarter,
                                              uint32_t tbase, bool live_tile, int ch, Stage& sg) {
  const int row0 = tc.m0 + quarter * 32;
  if (!live_tile || row0 >= min(pr.M, pr.e.rows_valid)) return;  // warp-uniform
  const bool split = pr.e.nsplit > 1;
  switch (pr.epi) {
    case EPI_AQ:
      if (split) epilogue_body<BN, EPI_AQ, true>(pr, tc, quarter, tbase, ch, sg);
      else epilogue_body<BN, EPI_AQ, false>(pr, tc, quarter, tbase, ch, sg);
      break;
    case EPI_HKG:
      if (split) epilogue_body<BN, EPI_HKG, true>(pr, tc, quarter, tbase, ch, sg);
      else epilogue_body<BN, EPI_HKG, false>(pr, tc, quarter, tbase, ch, sg);
      break;
    case EPI_GRAD:
      epilogue_body<BN, EPI_GRAD, false>(pr, tc, quarter, tbase, ch, sg);
      break;
    default:
      if (pr.e.out_bf16) epilogue_body<BN, EPI_Y, false>(pr, tc, quarter, tbase, ch, sg);
      else epilogue_body<BN, EPI_Y, true>(pr, tc, quarter, tbase, ch, sg);
      break;
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
  // launched as a programmatic dependent of the previous kernel of the
  // stream: the prologue above overlaps its tail; wait for its results here
  pdl_wait();
  pdl_trigger();

  int* const status = P.status;

  // The producer and the MMA issuer are single threads on the critical path:
  // per pass (one segment, or the two segments of a pair) they copy what they
  // need from the problem into registers, because every asm statement below
  // clobbers memory and would make the compiler re-read parameter space.
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
        const int tn = pr.tn, n0 = tc.n0 * tn, m0 = tc.m0, pair = pr.pair, nseg = pr.nseg;
        // passes: one per segment, or one per product when its segments are paired
        const int npass = pair ? (pr.nseg2 ? 2 : 1) : nseg + pr.nseg2;
        for (int ps = 0; ps < npass && ok; ++ps) {
          const bool second = pair ? ps == 1 : ps >= nseg;
          const int s0 = pair ? 0 : (second ? ps - nseg : ps);
          const Operand& A = second ? pr.a2 : pr.a;
          const Operand& B = second ? pr.b2 : pr.b;
          const int* sa = second ? pr.seg2_a : pr.seg_a;
          const int* sb = second ? pr.seg2_b : pr.seg_b;
          const CUtensorMap* const am = &A.map[sa[s0]];
          const CUtensorMap* const bm = &B.map[sb[s0]];
          // the other part of a pair: B lo (pair 1) or A lo (pair 2)
          const CUtensorMap* const m1 = pair == 1 ? &B.map[sb[1]] : &A.map[sa[1]];
          const int a_mn = A.mn_major, b_mn = B.mn_major, arow = A.row0, brow = B.row0;
          const int bn = second ? tn / 2 : tn;   // B rows (columns of this product)
          const int bn0 = second ? n0 / 2 : n0;
          const int bbytes = bn * BK * 2;
          const int na = pair == 2 ? 2 : 1, nb = pair == 1 ? 2 : 1;
          const uint32_t tx = (uint32_t)(na * BM * BK * 2 + nb * bbytes);
          const int az2 = tc.z % A.zdiv, az3 = tc.z / A.zdiv, bz2 = tc.z % B.zdiv,
                    bz3 = tc.z / B.zdiv;
          // TMA x coordinates are multiples of 8 bf16 (16 bytes) and the pass's
          // boxes fit the stage's A and B slots
          if (!TTT_BOUNDS((m0 & 7) == 0 && (bn0 & 7) == 0 && (kb0 * BK & 7) == 0 &&
                              nb * bbytes + (na - 1) * BM * BK * 2 <= BN * BK * 2 && bn <= BN &&
                              tc.z < pr.nz,
                          status)) {
            ok = false;
            break;
          }
          for (int kb = kb0; kb < kb0 + nk; ++kb, ++it) {
            const int st = it % kStages;
            if (it >= kStages && !mbar_wait(&sm.empty[st], ((it / kStages) - 1) & 1, status)) {
              ok = false;
              break;
            }
            const int k = kb * BK;
            uint64_t* const full = &sm.full[st];
            mbar_arrive_expect_tx(full, tx);
            for (int x = 0; x < na; ++x) {  // A, then A lo of a pair at b + bbytes
              uint8_t* const dst = x ? sm.b[st] + bbytes : sm.a[st];
              const CUtensorMap* const map = x ? m1 : am;
              if (!a_mn) {
                tma_load_4d(dst, map, full, k, arow + m0, az2, az3);
              } else {
                tma_load_4d(dst, map, full, m0, arow + k, az2, az3);
                tma_load_4d(dst + 8192, map, full, m0 + 64, arow + k, az2, az3);
              }
            }
            for (int x = 0; x < nb; ++x) {  // B, then B lo of a pair at b + bbytes
              uint8_t* const dst = sm.b[st] + (x ? bbytes : 0);
              const CUtensorMap* const map = x ? m1 : bm;
              if (!b_mn) {
                tma_load_4d(dst, map, full, k, brow + bn0, bz2, bz3);
              } else {
                for (int y = 0; y < bn / 64; ++y)
                  tma_load_4d(dst + y * 8192, map, full, bn0 + 64 * y, brow + k, bz2, bz3);
              }
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
        const int tn = pr.tn, pair = pr.pair, nseg = pr.nseg;
        const int npass = pair ? (pr.nseg2 ? 2 : 1) : nseg + pr.nseg2;
        const int ab = lt & 1;
        if (lt >= 2 && !mbar_wait(&sm.acc_empty[ab], ((lt >> 1) - 1) & 1, status)) break;
        umma::fence_after();
        const uint32_t dacc = tmem + ab * BN;
        for (int ps = 0; ps < npass && ok; ++ps) {
          const bool second = pair ? ps == 1 : ps >= nseg;
          const int a_mn = (second ? pr.a2 : pr.a).mn_major;
          const int b_mn = (second ? pr.b2 : pr.b).mn_major;
          const int bn = second ? tn / 2 : tn;
          const uint32_t bpart = (uint32_t)(bn * BK * 2) >> 4;  // offset of a pair's second part, 16 B units
          const uint32_t d = dacc + (second ? tn : 0);
          const uint32_t idesc = umma::instr_desc(1, BM, bn, a_mn, b_mn);
          // descriptors: fixed fields | start address, K steps of 16 as address
          // increments (2 KB for an MN-major operand, 32 B for a K-major one)
          const uint64_t abase = a_mn ? umma::smem_desc_base(8192, 1024) : umma::smem_desc_base(16, 1024);
          const uint64_t bbase = b_mn ? umma::smem_desc_base(8192, 1024) : umma::smem_desc_base(16, 1024);
          const uint32_t astep = a_mn ? 128u : 2u, bstep = b_mn ? 128u : 2u;
          // the accumulator (region) starts at zero with the product's first MMA
          const bool first = pair || ps == 0 || ps == nseg;
          for (int i = 0; i < nk; ++i, ++it) {
            const int st = it % kStages;
            if (!mbar_wait(&sm.full[st], (it / kStages) & 1, status)) {
              ok = false;
              break;
            }
            umma::fence_after();
            const uint32_t sa = (smem_u32(sm.a[st]) >> 4) & 0x3FFF;
            const uint32_t sb = (smem_u32(sm.b[st]) >> 4) & 0x3FFF;
            const uint64_t ad = abase | sa, bd = bbase | sb;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma::mma_bf16(d, ad + kk * astep, bd + kk * bstep, idesc,
                             (!first || i > 0 || kk > 0) ? 1u : 0u);
            if (pair) {  // the second part: A with B lo (pair 1) or A lo with B (pair 2)
              const uint64_t ad1 = pair == 2 ? abase | (sb + bpart) : ad;
              const uint64_t bd1 = pair == 1 ? bbase | (sb + bpart) : bd;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma::mma_bf16(d, ad1 + kk * astep, bd1 + kk * bstep, idesc, 1u);
            }
            umma::commit(&sm.empty[st]);
          }
        }
        if (!ok) break;
        umma::commit(&sm.acc_full[ab]);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9 ----------------
    const int quarter = warp & 3;
    const int ch = (warp - 2) >> 2;       // column half
    Stage sgr{sm.ostage[warp - 2], lane, false, status};
    int lt = 0;
    for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++lt) {
      const TileCoord tc = decode_tile(P, t);
      const Problem& pr = P.p[tc.pi];
      int kb0, nk;
      k_range(pr, tc.ks, kb0, nk);
      const int ab = lt & 1;
      const bool waited = mbar_wait(&sm.acc_full[ab], (lt >> 1) & 1, status);
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
