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
// S^T is a 128 x 128 fp32 accumulator in tensor memory for the whole sequence:
// the ΔS MMA accumulates into it, and the output MMA reads it directly as its
// A operand (kind::tf32, A from TMEM), so the state never leaves tensor memory
// and the sequential dependence stays inside the in-order MMA pipe.
//
// One CTA per (batch, head), 16 warps:
//   warp 0      TMA producer: Q tiles into a 2-slot ring (released once the
//               score MMA and the fp32 conversion have read them), K and V
//               tiles into a 3-stage ring (released when the tile's MMAs are
//               done), L2 prefetch further ahead; eta to smem
//   warp 1      TMEM owner; one thread issues all tcgen05.mma
//   warps 2-7   converters: fp32 copy of Q (the tf32 B operand)
//   warps 8-11  score epilogue: P = tril(scores) -> bf16 smem, Vt = eta * V in place
//   warps 12-15 output epilogue: S^T init from W0, Y tiles (staged in smem, then
//               stored as 16-byte row pieces), W_final
// Every barrier wait is bounded (%globaltimer); a timeout is recorded in the
// device status word and the kernel returns.
#include "common.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace ttt {
namespace {

constexpr int D = 128;         // dk = dv
constexpr int TT = 64;         // tokens per tile
constexpr int kStages = 3;     // Q/K/V ring
constexpr int kThreads = 512;
constexpr int kConvWarps = 6;
constexpr int kEpiWarp0 = 8;    // score epilogue warps 8-11
constexpr int kOutWarp0 = 12;   // output epilogue warps 12-15
constexpr int kL2Ahead = 4;    // tiles prefetched into L2 ahead of the smem ring
constexpr uint32_t kTileBytes = TT * D * 2;   // one bf16 [64 x 128] tile, 16 KB

// TMEM columns: S^T [0,128), scores [128,256) (2 x 64), Y^T [256,384) (2 x 64)
constexpr uint32_t kColS = 0, kColSc = 128, kColY = 256, kTmemCols = 512;

struct Smem {
  alignas(1024) uint8_t q[2][kTileBytes];          // Q ring, 2 boxes [64 t][64 d], 128B swizzle
  alignas(1024) uint8_t k[kStages][kTileBytes];    // K/V ring
  alignas(1024) uint8_t v[kStages][kTileBytes];    // becomes eta * V in place
  alignas(1024) uint8_t q32[2][TT * D * 4];        // 4 boxes [64 t][32 d] fp32
  alignas(1024) uint8_t p[2][TT * TT * 2];         // [64 t][64 i] bf16, 128B swizzle
  alignas(1024) __nv_bfloat16 ystage[TT * D];      // output tile [t][dv]
  float eta[kStages][TT];
  uint64_t full_q[2], q_free[2], full[kStages], conv[kStages], stage_free[kStages];
  uint64_t sc_full[2], p_ready[2], y_full[2], y_free[2], done;
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

__global__ void __launch_bounds__(kThreads, 1) la_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int ntiles = (p.T + TT - 1) / TT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.conv[s], kConvWarps);
      mbar_init(&sm.stage_free[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.full_q[x], 1);
      mbar_init(&sm.q_free[x], 1 + kConvWarps);  // score MMAs done + every converter warp
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.sc_full[x], 1);
      mbar_init(&sm.p_ready[x], 4);
      mbar_init(&sm.y_full[x], 1);
      mbar_init(&sm.y_free[x], 4);
    }
    mbar_init(&sm.done, 1);
    fence_mbar_init();
  }
  if (warp == 1) umma::tmem_alloc(&sm.tmem_base, kTmemCols);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sm.tmem_base;

  // S^T <- W0^T (output warps; lane = dv row r, columns = dk)
  if (warp >= kOutWarp0) {
    const int q4 = warp & 3, r = q4 * 32 + lane;
    const float* W0 = p.W0 + b * p.w0_sb + (int64_t)h * D * D;
    for (int c = 0; c < D; c += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = W0[(int64_t)(c + u) * D + r];
      umma::tmem_st16(tmem + ((uint32_t)(q4 * 32) << 16) + kColS + c, v);
    }
  }
  umma::fence_before();
  __syncthreads();
  umma::fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
    }
    const float* eta = p.eta.p + b * p.eta.sb + h * p.eta.sh;
    if (lane == 0)
      for (int j = 0; j < kL2Ahead && j < ntiles; ++j)
        for (int x = 0; x < 2; ++x) {
          tma_prefetch_l2_4d(&p.tq, 64 * x, j * TT, h, b);
          tma_prefetch_l2_4d(&p.tk, 64 * x, j * TT, h, b);
          tma_prefetch_l2_4d(&p.tv, 64 * x, j * TT, h, b);
        }
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kStages;
      if (lane == 0 && j + kL2Ahead < ntiles)
        for (int x = 0; x < 2; ++x) {
          tma_prefetch_l2_4d(&p.tq, 64 * x, (j + kL2Ahead) * TT, h, b);
          tma_prefetch_l2_4d(&p.tk, 64 * x, (j + kL2Ahead) * TT, h, b);
          tma_prefetch_l2_4d(&p.tv, 64 * x, (j + kL2Ahead) * TT, h, b);
        }
      const int t0 = j * TT;
      const int xq = j & 1;
      if (j >= 2 && !mbar_wait(&sm.q_free[xq], ((j >> 1) - 1) & 1, p.status)) return;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.full_q[xq], kTileBytes);
        for (int x = 0; x < 2; ++x)
          tma_load_4d(sm.q[xq] + x * 8192, &p.tq, &sm.full_q[xq], 64 * x, t0, h, b);
      }
      if (j >= kStages && !mbar_wait(&sm.stage_free[s], ((j / kStages) - 1) & 1, p.status))
        return;
      for (int i = lane; i < TT; i += 32)
        sm.eta[s][i] = (t0 + i < p.T) ? eta[(int64_t)(t0 + i) * p.eta.st] : 0.f;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.full[s], 2 * kTileBytes);
        for (int x = 0; x < 2; ++x) {
          tma_load_4d(sm.k[s] + x * 8192, &p.tk, &sm.full[s], 64 * x, t0, h, b);
          tma_load_4d(sm.v[s] + x * 8192, &p.tv, &sm.full[s], 64 * x, t0, h, b);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_sc = umma::instr_desc(1, TT, TT, 0, 0);    // Q K^T
      const uint32_t id_yq = umma::instr_desc(2, D, TT, 0, 0);     // S^T Q^T (tf32, A in TMEM)
      const uint32_t id_yp = umma::instr_desc(1, D, TT, 1, 0);     // Vt^T P^T
      const uint32_t id_ds = umma::instr_desc(1, D, D, 1, 1);      // Vt^T K
      auto issue_scores = [&](int j, bool block) -> int {  // 1 issued, 0 not ready, -1 timeout
        const int s = j % kStages;
        if (block) {
          if (!mbar_wait(&sm.full[s], (j / kStages) & 1, p.status) ||
              !mbar_wait(&sm.full_q[j & 1], (j >> 1) & 1, p.status))
            return -1;
        } else if (!mbar_try_wait(&sm.full[s], (j / kStages) & 1) ||
                   !mbar_try_wait(&sm.full_q[j & 1], (j >> 1) & 1)) {
          return 0;
        }
        umma::fence_after();
        const uint32_t qa = smem_u32(sm.q[j & 1]), ka = smem_u32(sm.k[s]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma::mma_bf16(tmem + kColSc + (j & 1) * TT, umma::smem_desc(qa + off, 16, 1024),
                         umma::smem_desc(ka + off, 16, 1024), id_sc, kk > 0);
        }
        umma::commit(&sm.sc_full[j & 1]);
        umma::commit(&sm.q_free[j & 1]);
        return 1;
      };
      bool ok = true;
      int issued = 0;  // score tiles issued so far
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j % kStages, x = j & 1;
        // the epilogue needs scores of tiles j and j+1 in flight
        while (ok && issued < j + 2 && issued < ntiles) {
          ok = issue_scores(issued, true) > 0;
          ++issued;
        }
        if (!ok) break;
        ok = mbar_wait(&sm.p_ready[x], (j >> 1) & 1, p.status) &&
             mbar_wait(&sm.conv[s], (j / kStages) & 1, p.status) &&
             (j < 2 || mbar_wait(&sm.y_free[x], ((j - 2) >> 1) & 1, p.status));
        if (!ok) break;
        umma::fence_after();
        const uint32_t dY = tmem + kColY + x * TT;
        const uint32_t q32 = smem_u32(sm.q32[x]), va = smem_u32(sm.v[s]),
                       pa = smem_u32(sm.p[x]), ka = smem_u32(sm.k[s]);
        // Y^T = S^T Q^T   (tf32, K = 128 in steps of 8; Q32 boxes of 32 columns)
#pragma unroll
        for (int kk = 0; kk < D / 8; ++kk)
          umma::mma_tf32_tmem_a(dY, tmem + kColS + 8 * kk,
                                umma::smem_desc(q32 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                id_yq, kk > 0);
        // Y^T += Vt^T P^T   (K = 64 tokens i)
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk)
          umma::mma_bf16(dY, umma::smem_desc(va + kk * 2048, 8192, 1024),
                         umma::smem_desc(pa + kk * 32, 16, 1024), id_yp, 1);
        // S^T += Vt^T K   (K = 64 tokens)
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk)
          umma::mma_bf16(tmem + kColS, umma::smem_desc(va + kk * 2048, 8192, 1024),
                         umma::smem_desc(ka + kk * 2048, 8192, 1024), id_ds, 1);
        umma::commit(&sm.y_full[x]);
        umma::commit(&sm.stage_free[s]);
        if (issued == j + 2 && issued < ntiles) {
          const int r = issue_scores(issued, false);
          if (r < 0) ok = false;
          issued += r > 0;
        }
      }
      umma::commit(&sm.done);
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - 64;  // 0 .. 32*kConvWarps-1
    constexpr int NC = 32 * kConvWarps;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kStages, x = j & 1;
      if (!mbar_wait(&sm.full_q[x], (j >> 1) & 1, p.status)) return;
      // the fp32-Q buffer of tile j-2 is free once that tile's MMAs are done
      if (j >= 2 && !mbar_wait(&sm.y_full[x], ((j - 2) >> 1) & 1, p.status)) return;
      // Q (bf16, 2 boxes of 64 cols) -> Q32 (fp32, 4 boxes of 32 cols): 8 columns per item
      for (int it = ct; it < TT * 16; it += NC) {
        const int r = it >> 4, g = it & 15;   // row, group of 8 columns
        const int col = g * 8;
        const uint4 a = *reinterpret_cast<const uint4*>(sm.q[x] + (col >> 6) * 8192 +
                                                        swz(r, (col & 63) >> 3));
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        float4 lo, hi;
        lo.x = __uint_as_float(w[0] << 16);
        lo.y = __uint_as_float(w[0] & 0xffff0000u);
        lo.z = __uint_as_float(w[1] << 16);
        lo.w = __uint_as_float(w[1] & 0xffff0000u);
        hi.x = __uint_as_float(w[2] << 16);
        hi.y = __uint_as_float(w[2] & 0xffff0000u);
        hi.z = __uint_as_float(w[3] << 16);
        hi.w = __uint_as_float(w[3] & 0xffff0000u);
        uint8_t* dst = sm.q32[x] + (col >> 5) * 8192;
        const int d16 = (col & 31) >> 2;
        *reinterpret_cast<float4*>(dst + swz(r, d16)) = lo;
        *reinterpret_cast<float4*>(dst + swz(r, d16 + 1)) = hi;
      }
      umma::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.conv[s]);
        mbar_arrive(&sm.q_free[x]);
      }
    }
  } else if (warp < kOutWarp0) {
    // ------------------------------------------------------------ score epilogue
    const int q4 = warp & 3;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    for (int j = 0; j < ntiles; ++j) {
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
          __align__(16) __nv_bfloat16 o[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) o[u] = __float2bfloat16_rn((c + u <= t) ? v[u] : 0.f);
          *reinterpret_cast<uint4*>(prow + swz(t, c >> 3)) = reinterpret_cast<uint4*>(o)[0];
          *reinterpret_cast<uint4*>(prow + swz(t, (c >> 3) + 1)) = reinterpret_cast<uint4*>(o)[1];
        }
      }
      // Vt = eta * V in place (stage j % kStages; its data landed before the scores)
      {
        const int s = j % kStages;
        const int ti = threadIdx.x - 32 * kEpiWarp0;  // 0..127
        for (int it = ti; it < TT * 16; it += 128) {
          const int r = it >> 4, c = it & 15;  // row, 16-byte chunk
          uint8_t* ptr = sm.v[s] + (c >> 3) * 8192 + swz(r, c & 7);
          uint4 a = *reinterpret_cast<uint4*>(ptr);
          const float er = sm.eta[s][r];
          uint32_t* w = reinterpret_cast<uint32_t*>(&a);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            __nv_bfloat162 v2 = __floats2bfloat162_rn(er * __uint_as_float(w[u] << 16),
                                                      er * __uint_as_float(w[u] & 0xffff0000u));
            w[u] = *reinterpret_cast<uint32_t*>(&v2);
          }
          *reinterpret_cast<uint4*>(ptr) = a;
        }
      }
      umma::fence_before();
      umma::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_ready[x]);
    }
  } else {
    // ------------------------------------------------------------ output epilogue
    const int q4 = warp & 3;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    auto do_y = [&](int j) -> bool {
      const int x = j & 1;
      const bool ok = mbar_wait(&sm.y_full[x], (j >> 1) & 1, p.status);
      umma::fence_after();
      const int r = q4 * 32 + lane;  // dv row
      const int t0 = j * TT;
      __nv_bfloat16* st = sm.ystage;
      for (int c = 0; c < TT && ok; c += 16) {
        float v[16];
        umma::tmem_ld16(tmem + lane_base + kColY + x * TT + c, v);
#pragma unroll
        for (int u = 0; u < 16; ++u) st[(c + u) * D + r] = __float2bfloat16_rn(v[u]);
      }
      umma::fence_before();
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the 4 output warps
      if (lane == 0) mbar_arrive(&sm.y_free[x]);       // TMEM tile read
      // 64 rows x 256 bytes: each thread stores 16-byte pieces of whole rows
      const int ti = threadIdx.x - 32 * kOutWarp0;  // 0..127
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out.p) + b * p.out.sb + h * p.out.sh;
      for (int it = ti; it < TT * 16 && ok; it += 128) {
        const int t = it >> 4, c = it & 15;
        if (t0 + t < p.T)
          *reinterpret_cast<uint4*>(o + (int64_t)(t0 + t) * p.out.st + c * 8) =
              *reinterpret_cast<const uint4*>(st + t * D + c * 8);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // staging buffer free again
      return ok;
    };
    for (int j = 0; j < ntiles; ++j)
      if (!do_y(j)) return;
    // final state
    if (p.W_final) {
      if (!mbar_wait(&sm.done, 0, p.status)) return;
      umma::fence_after();
      const int r = q4 * 32 + lane;
      float* Wf = p.W_final + (int64_t)bh * D * D;
      for (int c = 0; c < D; c += 16) {
        float v[16];
        umma::tmem_ld16(tmem + lane_base + kColS + c, v);
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
  la_tc_kernel<<<a.B * a.H, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ttt
