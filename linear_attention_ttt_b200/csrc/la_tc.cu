// Inner-product-loss TTT layer (= causal linear attention with per-token
// weights) on the 5th-generation tensor cores, d = dk = dv = 128, bf16 tokens,
// fp32 state.
//
// "Test-Time Training (TTT)" summary, sections "Linear Attention" and
// "예시 1: Linear Attention 유도": with the inner-product loss the gradient
// -k^T v does not depend on W, so mini-batch GD with any chunk size gives
//   S_t = S_{t-1} + eta_t k_t^T v_t,   y_t = q_t S_t,   S_0 = W0.
// The kernel therefore walks each sequence in tiles of 64 tokens whatever the
// requested chunk, with (Q, K, V one tile, Vt = diag(eta) V, P = tril(Q K^T)):
//   Y^T = S^T Q^T + Vt^T P^T          (output tile, transposed)
//   S^T = S^T + Vt^T K                (state after the tile)
// Tensor memory (512 columns) holds, for the whole sequence:
//   S^T   fp32, 128 lanes x 128 columns: the exact state, accumulated by MMA;
//   S^T   bf16 copy (2 per column), the A operand of S^T Q^T, refreshed from
//         the fp32 state after each tile;
//   Vt^T  bf16 (2 per column), written per tile by the threads that scale V
//         by eta, the A operand of Vt^T P^T and of the state update;
//   the score tile Q K^T (2 buffers) and the output tile Y^T (2 buffers).
// The A operands come from tensor memory, so the only shared-memory operands
// are Q, K (from TMA) and P (written by the score warps).
//
// Each (batch, head) runs on two CTAs that split the sequence at tile `mid`
// (CTA 1 takes 7/16 of the tiles, rounded down).
// CTA 0 handles tiles [0, mid). CTA 1 first builds the state after tile mid-1
// with MMAs only: per tile, K scaled by eta in place and
// S^T += V^T (diag(eta) K) with both operands in shared memory. It then
// handles tiles [mid, end) with the full loop below and writes W_final.
//
// Per CTA, 16 warps:
//   warp 0      TMA producer: Q, K, V tiles into a 4-stage ring (plus L2
//               prefetch further ahead); eta to smem
//   warp 1      TMEM owner; one thread issues all tcgen05.mma
//   warps 4-7   Vt^T into tensor memory (eta * V, transposed by lane = dv)
//   warps 8-11  score epilogue: P = tril(scores) -> bf16 smem
//   warps 12-15 state/output warps: S^T init from W0, the bf16 refresh of S^T
//               after each tile, Y tiles (staged in smem, stored as 16-byte
//               row pieces), W_final
// Every barrier wait is bounded (%globaltimer); a timeout is recorded in the
// device status word and the kernel returns.
#include "common.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int D = 128;         // dk = dv
constexpr int TT = 64;         // tokens per tile
constexpr int kStages = 4;     // Q/K/V ring
constexpr int kThreads = 512;
constexpr int kVtWarp0 = 4, kScWarp0 = 8, kOutWarp0 = 12;
constexpr int kL2Ahead = 4;    // tiles prefetched into L2 ahead of the smem ring
// CTA 1's share of the tiles, in sixteenths (rounded down): it also rebuilds
// the state over CTA 0's tiles, so an even split leaves CTA 0 idle at the end
// (B4 H16 T4096: 7/16 111.5 us, 8/16 113.6 us, 6/16 114.1 us, 5/16 122.8 us).
constexpr int kSeg1Sixteenths = 7;
constexpr uint32_t kTileBytes = TT * D * 2;   // one bf16 [64 x 128] tile, 16 KB

// TMEM columns
constexpr uint32_t kColS = 0;      // S^T fp32            [0, 128)
constexpr uint32_t kColSb = 128;   // S^T bf16 pairs       [128, 192)
constexpr uint32_t kColSc = 192;   // scores, 2 x 64       [192, 320)
constexpr uint32_t kColY = 320;    // Y^T, 2 x 64          [320, 448)
constexpr uint32_t kColVt = 448;   // Vt^T bf16 pairs 2x32 [448, 512)
constexpr uint32_t kTmemCols = 512;

struct Smem {
  alignas(1024) uint8_t q[kStages][kTileBytes];    // 2 boxes [64 t][64 d], 128B swizzle
  alignas(1024) uint8_t k[kStages][kTileBytes];
  alignas(1024) uint8_t v[kStages][kTileBytes];
  alignas(1024) uint8_t p[2][TT * TT * 2];         // [64 t][64 i] bf16, 128B swizzle
  alignas(1024) __nv_bfloat16 ystage[TT * D];      // output tile [t][dv]
  float eta[kStages][TT];
  uint64_t full[kStages], stage_free[kStages];
  uint64_t sc_full[2], p_ready[2], vt_ready[2], y_full[2], y_free[2], s_ready, done;
  uint64_t k_scaled[2], p1_done;  // state-only prefix (second CTA of a head)
  uint32_t tmem_base;
};

struct Params {
  CUtensorMap tq, tk, tv;  // {128, T, H, B}, box {64, 64, 1, 1}
  EtaView eta;
  const float* W0;
  int64_t w0_sb;
  TokViewMut out;
  float* W_final;
  int B, H, T;
  int* status;
};

// byte offset of 16-byte chunk `c16` of row `r` in a 128B-swizzled box
__device__ __forceinline__ uint32_t swz(int r, int c16) {
  return r * 128 + ((c16 ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 32 lanes x 32 consecutive 32-bit TMEM columns from 32 registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// bf16 copy of the fp32 state row held by this lane (128 columns -> 64 pairs).
__device__ __forceinline__ void refresh_state_copy(uint32_t tmem_lane) {
  for (int half = 0; half < 2; ++half) {
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 64; c += 16) {
      float v[16];
      umma::tmem_ld16(tmem_lane + kColS + 64 * half + c, v);
#pragma unroll
      for (int u = 0; u < 16; u += 2) pk[(c + u) / 2] = pack2(v[u], v[u + 1]);
    }
    tmem_st32(tmem_lane + kColSb + 32 * half, pk);
  }
}

__global__ void __launch_bounds__(kThreads, 1) la_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x >> 1, seg = blockIdx.x & 1, b = bh / p.H, h = bh % p.H;
  if (!TTT_BOUNDS(bh < p.B * p.H, p.status)) return;  // uniform over both CTAs of the head
  const int ntot = (p.T + TT - 1) / TT, mid = ntot - (ntot * kSeg1Sixteenths) / 16;
  // tiles [0, p1) build the state only; tiles [p1, tend) run the full loop
  const int p1 = seg ? mid : 0, tend = seg ? ntot : mid, n2 = tend - p1;
  const int s0 = seg ? 1 : 0;  // s_ready phase of the first full tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.stage_free[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.sc_full[x], 1);
      mbar_init(&sm.p_ready[x], 4);
      mbar_init(&sm.vt_ready[x], 4);
      mbar_init(&sm.y_full[x], 1);
      mbar_init(&sm.y_free[x], 4);
    }
    mbar_init(&sm.s_ready, 4);
    mbar_init(&sm.done, 1);
    mbar_init(&sm.k_scaled[0], 4);
    mbar_init(&sm.k_scaled[1], 4);
    mbar_init(&sm.p1_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(&sm.tmem_base, kTmemCols);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sm.tmem_base;

  // S^T <- W0^T in fp32 and its bf16 copy (state warps; lane = dv row r)
  if (warp >= kOutWarp0) {
    const int q4 = warp & 3, r = q4 * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const float* W0 = p.W0 + b * p.w0_sb + (int64_t)h * D * D;
    for (int c = 0; c < D; c += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = W0[(int64_t)(c + u) * D + r];
      umma::tmem_st16(tl + kColS + c, v);
    }
    refresh_state_copy(tl);
    umma::fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.s_ready);  // phase 0: S_0
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      for (int j = 0; j < kL2Ahead && j < tend; ++j)
        for (int x = 0; x < 2; ++x) {
          if (j >= p1) tma_prefetch_l2_4d(&p.tq, 64 * x, j * TT, h, b);
          tma_prefetch_l2_4d(&p.tk, 64 * x, j * TT, h, b);
          tma_prefetch_l2_4d(&p.tv, 64 * x, j * TT, h, b);
        }
    }
    // Learning rates are loaded four tiles ahead into four register slots (2
    // values per lane per tile); the loop is unrolled by four so every slot
    // keeps a fixed register and is read only when its tile is issued.
    const float* eta = p.eta.p + b * p.eta.sb + h * p.eta.sh;
    auto load_eta = [&](int j, float& e0, float& e1) {
      const int t = j * TT + lane;
      e0 = (j < tend && t < p.T) ? eta[(int64_t)t * p.eta.st] : 0.f;
      e1 = (j < tend && t + 32 < p.T) ? eta[(int64_t)(t + 32) * p.eta.st] : 0.f;
    };
    float r0a, r0b, r1a, r1b, r2a, r2b, r3a, r3b;
    load_eta(0, r0a, r0b);
    load_eta(1, r1a, r1b);
    load_eta(2, r2a, r2b);
    load_eta(3, r3a, r3b);
    int j = 0;
    auto issue = [&](float& ea, float& eb) -> bool {
      if (j >= tend) return false;
      const int s = j % kStages;
      const bool full_tile = j >= p1;  // state-only tiles need no Q
      if (lane == 0 && j + kL2Ahead < tend)
        for (int x = 0; x < 2; ++x) {
          if (j + kL2Ahead >= p1) tma_prefetch_l2_4d(&p.tq, 64 * x, (j + kL2Ahead) * TT, h, b);
          tma_prefetch_l2_4d(&p.tk, 64 * x, (j + kL2Ahead) * TT, h, b);
          tma_prefetch_l2_4d(&p.tv, 64 * x, (j + kL2Ahead) * TT, h, b);
        }
      if (j >= kStages && !mbar_wait(&sm.stage_free[s], ((j / kStages) - 1) & 1, p.status))
        return false;
      const int t0 = j * TT;
      sm.eta[s][lane] = ea;
      sm.eta[s][lane + 32] = eb;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.full[s], (full_tile ? 3 : 2) * kTileBytes);
        for (int x = 0; x < 2; ++x) {
          if (full_tile) tma_load_4d(sm.q[s] + x * 8192, &p.tq, &sm.full[s], 64 * x, t0, h, b);
          tma_load_4d(sm.k[s] + x * 8192, &p.tk, &sm.full[s], 64 * x, t0, h, b);
          tma_load_4d(sm.v[s] + x * 8192, &p.tv, &sm.full[s], 64 * x, t0, h, b);
        }
      }
      load_eta(j + 4, ea, eb);
      ++j;
      return true;
    };
    while (issue(r0a, r0b) && issue(r1a, r1b) && issue(r2a, r2b) && issue(r3a, r3b)) {
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_sc = umma::instr_desc(1, TT, TT, 0, 0);   // Q K^T            (M=64)
      const uint32_t id_y = umma::instr_desc(1, D, TT, 0, 0);     // S^T Q^T, Vt^T P^T (A in TMEM)
      const uint32_t id_ds = umma::instr_desc(1, D, D, 0, 1);     // Vt^T K           (A in TMEM)
      auto issue_scores = [&](int j, bool block) -> int {  // 1 issued, 0 not ready, -1 timeout
        const int g = p1 + j, s = g % kStages;              // g: tile index in the sequence
        if (block) {
          if (!mbar_wait(&sm.full[s], (g / kStages) & 1, p.status)) return -1;
        } else if (!mbar_try_wait(&sm.full[s], (g / kStages) & 1)) {
          return 0;
        }
        umma::fence_after();
        const uint32_t qa = smem_u32(sm.q[s]), ka = smem_u32(sm.k[s]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma::mma_bf16(tmem + kColSc + (j & 1) * TT, umma::smem_desc(qa + off, 16, 1024),
                         umma::smem_desc(ka + off, 16, 1024), id_sc, kk > 0);
        }
        umma::commit(&sm.sc_full[j & 1]);
        return 1;
      };
      bool ok = true;
      // state-only prefix: S^T += V^T (diag(eta) K), both operands MN-major
      if (p1 > 0) {
        const uint32_t id_p1 = umma::instr_desc(1, D, D, 1, 1);
        ok = mbar_wait(&sm.s_ready, 0, p.status);  // S^T holds W0^T
        for (int j = 0; j < p1 && ok; ++j) {
          const int s = j % kStages;
          ok = mbar_wait(&sm.full[s], (j / kStages) & 1, p.status) &&
               mbar_wait(&sm.k_scaled[j & 1], (j >> 1) & 1, p.status);
          if (!ok) break;
          umma::fence_after();
          const uint32_t va = smem_u32(sm.v[s]), ka = smem_u32(sm.k[s]);
#pragma unroll
          for (int kk = 0; kk < TT / 16; ++kk)
            umma::mma_bf16(tmem + kColS, umma::smem_desc(va + kk * 2048, 8192, 1024),
                           umma::smem_desc(ka + kk * 2048, 8192, 1024), id_p1, 1);
          umma::commit(&sm.stage_free[s]);
        }
        umma::commit(&sm.p1_done);
      }
      int issued = 0;  // score tiles issued so far (counted from p1)
      for (int j = 0; j < n2 && ok; ++j) {
        const int g = p1 + j, s = g % kStages, x = j & 1;
        // the score epilogue needs the scores of tiles j and j+1 in flight
        while (ok && issued < j + 2 && issued < n2) {
          ok = issue_scores(issued, true) > 0;
          ++issued;
        }
        if (!ok) break;
        ok = mbar_wait(&sm.p_ready[x], (j >> 1) & 1, p.status) &&
             mbar_wait(&sm.vt_ready[x], (j >> 1) & 1, p.status) &&
             mbar_wait(&sm.s_ready, (s0 + j) & 1, p.status) &&
             (j < 2 || mbar_wait(&sm.y_free[x], ((j - 2) >> 1) & 1, p.status));
        if (!ok) break;
        umma::fence_after();
        const uint32_t dY = tmem + kColY + x * TT;
        const uint32_t vt = tmem + kColVt + x * 32;
        const uint32_t qa = smem_u32(sm.q[s]), pa = smem_u32(sm.p[x]), ka = smem_u32(sm.k[s]);
        // Y^T = S^T Q^T   (A = bf16 state copy in TMEM, K = 128 in steps of 16)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma::mma_bf16_tmem_a(dY, tmem + kColSb + 8 * kk,
                                umma::smem_desc(qa + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                id_y, kk > 0);
        // Y^T += Vt^T P^T   (K = 64 tokens i)
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk)
          umma::mma_bf16_tmem_a(dY, vt + 8 * kk, umma::smem_desc(pa + kk * 32, 16, 1024), id_y, 1);
        // S^T += Vt^T K   (K = 64 tokens; K tile read MN-major)
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk)
          umma::mma_bf16_tmem_a(tmem + kColS, vt + 8 * kk,
                                umma::smem_desc(ka + kk * 2048, 8192, 1024), id_ds, 1);
        umma::commit(&sm.y_full[x]);
        umma::commit(&sm.stage_free[s]);
        if (issued == j + 2 && issued < n2) {
          const int r = issue_scores(issued, false);
          if (r < 0) ok = false;
          issued += r > 0;
        }
      }
      umma::commit(&sm.done);
    }
  } else if (warp >= kVtWarp0 && warp < kScWarp0) {
    // ------------------------------------------------------------ Vt^T -> TMEM
    const int q4 = warp & 3, r = q4 * 32 + lane;   // dv row
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    // column r of the V tile: box r / 64, 16-byte chunk (r % 64) / 8, byte 2 * (r % 8)
    const uint32_t box = (uint32_t)(r >> 6) * 8192, chunk = (r & 63) >> 3, byte = (r & 7) * 2;
    // state-only prefix: K rows scaled by eta in place (8 x 16 bytes per thread)
    const int ti = threadIdx.x - 32 * kVtWarp0;  // 0..127
    for (int j = 0; j < p1; ++j) {
      const int s = j % kStages;
      if (!mbar_wait(&sm.full[s], (j / kStages) & 1, p.status)) return;
      // k_scaled[j & 1] is free again once tile j-2's MMAs have completed
      // (they released that tile's stage)
      if (j >= 2 && !mbar_wait(&sm.stage_free[(j - 2) % kStages], ((j - 2) / kStages) & 1, p.status))
        return;
      const float* et = sm.eta[s];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int c = ti + 128 * m;                 // 16-byte chunk of the K tile
        const int t = (c & 511) >> 3;               // its row (token)
        uint4* ptr = reinterpret_cast<uint4*>(sm.k[s] + (c >> 9) * 8192 + t * 128 + (c & 7) * 16);
        uint4 u = *ptr;
        uint32_t* w = reinterpret_cast<uint32_t*>(&u);
        const float e = et[t];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 x2 = *reinterpret_cast<const __nv_bfloat162*>(&w[q]);
          w[q] = pack2(e * __low2float(x2), e * __high2float(x2));
        }
        *ptr = u;
      }
      umma::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.k_scaled[j & 1]);
    }
    for (int j = 0; j < n2; ++j) {
      const int g = p1 + j, s = g % kStages, x = j & 1;
      if (!mbar_wait(&sm.full[s], (g / kStages) & 1, p.status)) return;
      // the Vt^T buffer of tile j-2 is free once that tile's MMAs are done
      if (j >= 2 && !mbar_wait(&sm.y_full[x], ((j - 2) >> 1) & 1, p.status)) return;
      const uint8_t* vb = sm.v[s] + box + byte;
      const float* et = sm.eta[s];
      uint32_t pk[32];
#pragma unroll 8
      for (int i = 0; i < TT; i += 2) {
        const float v0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vb + swz(i, chunk)));
        const float v1 =
            __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vb + swz(i + 1, chunk)));
        pk[i >> 1] = pack2(et[i] * v0, et[i + 1] * v1);
      }
      tmem_st32(tl + kColVt + x * 32, pk);
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.vt_ready[x]);
    }
  } else if (warp >= kScWarp0 && warp < kOutWarp0) {
    // ------------------------------------------------------------ score epilogue
    const int q4 = warp & 3;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    for (int j = 0; j < n2; ++j) {
      const int x = j & 1;
      if (!mbar_wait(&sm.sc_full[x], (j >> 1) & 1, p.status)) return;
      umma::fence_after();
      // score tile (M = 64): row t = 16*q4 + lane lives in lane (q4*32 + lane) for lane < 16
      const int t = 16 * q4 + lane;
      uint8_t* prow = sm.p[x];
      for (int c = 0; c < TT; c += 16) {
        float v[16];
        umma::tmem_ld16(tmem + lane_base + kColSc + x * TT + c, v);
        if (lane < 16) {
          uint4 o[2];
          uint32_t* ow = reinterpret_cast<uint32_t*>(o);
#pragma unroll
          for (int u = 0; u < 16; u += 2)
            ow[u / 2] = pack2((c + u <= t) ? v[u] : 0.f, (c + u + 1 <= t) ? v[u + 1] : 0.f);
          *reinterpret_cast<uint4*>(prow + swz(t, c >> 3)) = o[0];
          *reinterpret_cast<uint4*>(prow + swz(t, (c >> 3) + 1)) = o[1];
        }
      }
      umma::fence_before();
      umma::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_ready[x]);
    }
  } else if (warp >= kOutWarp0) {
    // ------------------------------------------------------------ state / output
    const int q4 = warp & 3;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const int r = q4 * 32 + lane;  // dv row
    if (p1 > 0) {
      // the state after the prefix, copied to bf16 for the first full tile
      if (!mbar_wait(&sm.p1_done, 0, p.status)) return;
      umma::fence_after();
      refresh_state_copy(tl);
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_ready);  // phase 1
    }
    for (int j = 0; j < n2; ++j) {
      const int x = j & 1;
      // On a timeout the warp still takes part in both named barriers below.
      const bool ok = mbar_wait(&sm.y_full[x], (j >> 1) & 1, p.status);
      umma::fence_after();
      // 1) bf16 copy of the updated state for the next tile's S^T Q^T
      if (ok && j + 1 < n2) {
        refresh_state_copy(tl);
        umma::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_ready);
      }
      // 2) Y^T tile -> [t][dv] bf16 staging -> 16-byte row pieces
      const int t0 = (p1 + j) * TT;
      __nv_bfloat16* st = sm.ystage;
      for (int c = 0; c < TT && ok; c += 16) {
        float v[16];
        umma::tmem_ld16(tl + kColY + x * TT + c, v);
#pragma unroll
        for (int u = 0; u < 16; ++u) st[(c + u) * D + r] = __float2bfloat16_rn(v[u]);
      }
      umma::fence_before();
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the 4 state/output warps
      if (lane == 0) mbar_arrive(&sm.y_free[x]);       // TMEM tile read
      const int ti = threadIdx.x - 32 * kOutWarp0;     // 0..127
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out.p) + b * p.out.sb + h * p.out.sh;
      for (int it = ti; it < TT * 16 && ok; it += 128) {
        const int tt = it >> 4, c = it & 15;
        if (t0 + tt < p.T && TTT_BOUNDS(tt < TT && c * 8 + 8 <= D, p.status))
          *reinterpret_cast<uint4*>(o + (int64_t)(t0 + tt) * p.out.st + c * 8) =
              *reinterpret_cast<const uint4*>(st + tt * D + c * 8);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // staging buffer free again
      if (!ok) return;
    }
    // final state
    if (p.W_final && seg == 1) {
      if (!mbar_wait(&sm.done, 0, p.status)) return;
      umma::fence_after();
      float* Wf = p.W_final + (int64_t)bh * D * D;
      for (int c = 0; c < D; c += 16) {
        float v[16];
        umma::tmem_ld16(tl + kColS + c, v);
#pragma unroll
        for (int u = 0; u < 16; ++u) Wf[(int64_t)(c + u) * D + r] = v[u];
      }
    }
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) umma::tmem_dealloc(tmem, kTmemCols);
}

bool token_map(CUtensorMap* m, const TokView& v, int B, int H, int T) {
  TokView x = v;
  if (B == 1) x.sb = (int64_t)H * T * D;
  if (H == 1) x.sh = (int64_t)T * D;
  if (T == 1) x.st = D;
  uint64_t dims[4] = {(uint64_t)D, (uint64_t)T, (uint64_t)H, (uint64_t)B};
  uint64_t strides[3] = {(uint64_t)x.st * 2, (uint64_t)x.sh * 2, (uint64_t)x.sb * 2};
  uint32_t box[4] = {64, TT, 1, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x.p, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool la_tc_supported(const LinearArgs& a) {
  return a.loss == TTT_LOSS_NEG_DOT && a.dk == D && a.dv == D && a.T > 0;
}

cudaError_t launch_la_tc(const LinearArgs& a, cudaStream_t s) {
  Params p;
  if (!token_map(&p.tq, a.q, a.B, a.H, a.T) || !token_map(&p.tk, a.k, a.B, a.H, a.T) ||
      !token_map(&p.tv, a.v, a.B, a.H, a.T))
    return cudaErrorInvalidValue;
  p.eta = a.eta;
  p.W0 = a.W0;
  p.w0_sb = a.w0_sb;
  p.out = a.out;
  p.W_final = a.W_final;
  p.B = a.B;
  p.H = a.H;
  p.T = a.T;
  p.status = a.status;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(la_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  la_tc_kernel<<<a.B * a.H * 2, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ttt
