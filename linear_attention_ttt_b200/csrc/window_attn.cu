// Sliding-window causal softmax attention, the attention half of LaCT's
// hybrid block ("Test-Time Training Done Right" review, sections 3.1 and 4:
// window attention models the relations between tokens in a fixed range,
// and attention and the TTT layer share Q, K, V with their outputs
// combined). For every token t:
//   y_t = sum_{t-w < i <= t} softmax_i(q_t . k_i / sqrt(d)) v_i.
//
// Layout: one CTA of eight warps per 128 query rows of one (batch, head);
// each warp owns 16 query rows and keeps their Q fragments in registers (in
// shared memory for d = 256). Key/value tiles of 64 tokens covering the
// window of the CTA's rows stream through two shared-memory buffers with
// cp.async (the next tile loads while the current one is used), stored as
// 128-byte-swizzled 64-column panels; S = Q K^T and O += P V run on mma.sync
// m16n8k16 (bf16 operands, fp32 accumulation) with an online softmax in
// registers (running row maximum and sum, rescaling O when the maximum
// grows). Only tiles that cross a warp's causal or window edge are masked,
// and a warp skips tiles outside its rows' windows. With `accumulate` the
// result is added to what `out` holds (used to sum the attention output with
// the LaCT output).
#include "common.cuh"

namespace ttt {
namespace {

constexpr int kRows = 128;    // query rows per CTA (eight warps of 16)
constexpr int kKeys = 64;     // keys per tile
constexpr int kThreads = 256;

// byte offset of (row, col) in a [ROWS rows] x [D cols] bf16 tile stored as
// D/64 panels of [ROWS][64] with the 128-byte swizzle
template <int ROWS>
__device__ __forceinline__ uint32_t pofs(int row, int col) {
  return (col >> 6) * (ROWS * 128) + row * 128 + ((((col >> 3) & 7) ^ (row & 7)) << 4) +
         ((col & 7) << 1);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

struct WinParams {
  TokView q, k, v;
  TokViewMut out;
  int B, H, T, window, accumulate;
  float scale_log2;  // log2(e) / sqrt(d)
};

// ROWS rows x D columns of a token tensor into a swizzled tile with 16-byte
// cp.async copies (rows >= T read as zero); the caller commits the group.
template <int D, int ROWS>
__device__ __forceinline__ void load_tile_async(uint8_t* dst, const TokView& v, int b, int h,
                                                int t0, int T) {
  const __nv_bfloat16* base = static_cast<const __nv_bfloat16*>(v.p) + b * v.sb + h * v.sh;
  const uint32_t d0 = smem_u32(dst);
  constexpr int kChunks = ROWS * D / 8;
#pragma unroll 4
  for (int x = threadIdx.x; x < kChunks; x += kThreads) {
    const int r = x / (D / 8), c = (x % (D / 8)) * 8;
    const bool ok = t0 + r < T;
    const __nv_bfloat16* src = ok ? base + (int64_t)(t0 + r) * v.st + c : base;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d0 + pofs<ROWS>(r, c)),
                 "l"(src), "r"(ok ? 16 : 0)
                 : "memory");
  }
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads) window_attn_kernel(const __grid_constant__ WinParams p) {
  constexpr bool kQReg = D <= 128;   // Q fragments in registers
  constexpr int kTile = kKeys * D * 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sq = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* skv = sq + kRows * D * 2;  // [2 buffers][K tile, V tile]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c4 = lane & 3, mi = lane >> 3, rr = lane & 7;
  const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int q0 = blockIdx.x * kRows;
  const int r0 = warp * 16;
  const int row_a = q0 + r0 + g, row_b = row_a + 8;  // this thread's two query rows
  const int wmin = q0 + r0, wmax = wmin + 15;        // this warp's rows

  const int k_lo = max(0, q0 - p.window + 1);
  const int k_hi = min(p.T - 1, q0 + kRows - 1);
  const int kt0 = (k_lo / kKeys) * kKeys;
  const int ntiles = k_hi >= kt0 ? (k_hi - kt0) / kKeys + 1 : 0;

  load_tile_async<D, kRows>(sq, p.q, b, h, q0, p.T);
  cp_async_commit();
  if (ntiles > 0) {
    load_tile_async<D, kKeys>(skv, p.k, b, h, kt0, p.T);
    load_tile_async<D, kKeys>(skv + kTile, p.v, b, h, kt0, p.T);
  }
  cp_async_commit();

  const uint32_t qa = smem_u32(sq);
  uint32_t qf[kQReg ? D / 16 : 1][4];
  if constexpr (kQReg) {
    cp_async_wait<1>();  // the Q tile
    __syncthreads();
#pragma unroll
    for (int kb = 0; kb < D / 16; ++kb)
      ldsm4(qf[kb], qa + pofs<kRows>(r0 + rr + 8 * (mi & 1), 16 * kb + 8 * (mi >> 1)));
  }

  float O[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int j = 0; j < ntiles; ++j) {
    const int kt = kt0 + j * kKeys;
    // prefetch tile j + 1 into the other buffer (free: the barrier that ended
    // iteration j - 1 follows its last read)
    if (j + 1 < ntiles) {
      uint8_t* nb = skv + ((j + 1) & 1) * 2 * kTile;
      load_tile_async<D, kKeys>(nb, p.k, b, h, kt + kKeys, p.T);
      load_tile_async<D, kKeys>(nb + kTile, p.v, b, h, kt + kKeys, p.T);
    }
    cp_async_commit();
    cp_async_wait<1>();  // everything but the prefetch just issued
    __syncthreads();
    const uint32_t ka = smem_u32(skv + (j & 1) * 2 * kTile), va = ka + kTile;

    // this warp's rows see keys (row - window, row]: skip tiles outside, mask
    // only tiles that cross an edge (or hold keys beyond T)
    const bool skip = kt > wmax || kt + kKeys - 1 <= wmin - p.window;
    if (!skip) {
      const bool full = kt + kKeys - 1 <= wmin && kt > wmax - p.window && kt + kKeys <= p.T;
      float S[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) S[n][0] = S[n][1] = S[n][2] = S[n][3] = 0.f;
#pragma unroll
      for (int kb = 0; kb < D / 16; ++kb) {
        uint32_t a[4];
        if constexpr (kQReg) {
#pragma unroll
          for (int u = 0; u < 4; ++u) a[u] = qf[kb][u];
        } else {
          ldsm4(a, qa + pofs<kRows>(r0 + rr + 8 * (mi & 1), 16 * kb + 8 * (mi >> 1)));
        }
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t bk[4];
          ldsm4(bk, ka + pofs<kKeys>(16 * np + 8 * (mi >> 1) + rr, 16 * kb + 8 * (mi & 1)));
          mma_bf16(S[2 * np], a, bk[0], bk[1]);
          mma_bf16(S[2 * np + 1], a, bk[2], bk[3]);
        }
      }
      // mask (causal and window) where needed, scale to log2 units, online softmax
      float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int key = kt + 8 * n + 2 * c4 + (u & 1);
          const int row = (u < 2) ? row_a : row_b;
          const bool ok = full || (key <= row && key > row - p.window);
          S[n][u] = ok ? S[n][u] * p.scale_log2 : -INFINITY;
        }
        mx_a = fmaxf(mx_a, fmaxf(S[n][0], S[n][1]));
        mx_b = fmaxf(mx_b, fmaxf(S[n][2], S[n][3]));
      }
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, o));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, o));
      }
      const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
      // a row with no valid key so far keeps everything at zero
      const float base_a = mn_a == -INFINITY ? 0.f : mn_a;
      const float base_b = mn_b == -INFINITY ? 0.f : mn_b;
      const float al_a = exp2f(m_a - base_a), al_b = exp2f(m_b - base_b);
      m_a = mn_a;
      m_b = mn_b;
      float sum_a = 0.f, sum_b = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        S[n][0] = exp2f(S[n][0] - base_a);
        S[n][1] = exp2f(S[n][1] - base_a);
        S[n][2] = exp2f(S[n][2] - base_b);
        S[n][3] = exp2f(S[n][3] - base_b);
        sum_a += S[n][0] + S[n][1];
        sum_b += S[n][2] + S[n][3];
      }
      l_a = l_a * al_a + sum_a;
      l_b = l_b * al_b + sum_b;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        O[n][0] *= al_a;
        O[n][1] *= al_a;
        O[n][2] *= al_b;
        O[n][3] *= al_b;
      }
      // O += P V
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4];
        pa[0] = pack2(S[2 * kk][0], S[2 * kk][1]);
        pa[1] = pack2(S[2 * kk][2], S[2 * kk][3]);
        pa[2] = pack2(S[2 * kk + 1][0], S[2 * kk + 1][1]);
        pa[3] = pack2(S[2 * kk + 1][2], S[2 * kk + 1][3]);
#pragma unroll
        for (int jn = 0; jn < D / 8; jn += 2) {
          uint32_t r[4];
          ldsm4_t(r, va + pofs<kKeys>(16 * kk + rr + 8 * (mi & 1), 8 * (jn + (mi >> 1))));
          mma_bf16(O[jn], pa, r[0], r[1]);
          mma_bf16(O[jn + 1], pa, r[2], r[3]);
        }
      }
    }
    __syncthreads();  // buffer j & 1 is free for the prefetch of tile j + 2
  }
  cp_async_wait<0>();
  // the row sums were accumulated per thread over its own keys: reduce the quad
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, o);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, o);
  }
  const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f, inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(p.out.p) + b * p.out.sb + h * p.out.sh;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int c = 8 * n + 2 * c4;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = half ? row_b : row_a;
      if (row >= p.T) continue;
      float v0 = O[n][2 * half] * (half ? inv_b : inv_a);
      float v1 = O[n][2 * half + 1] * (half ? inv_b : inv_a);
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(ob + (int64_t)row * p.out.st + c);
      if (p.accumulate) {
        const float2 old = __bfloat1622float2(*dst);
        v0 += old.x;
        v1 += old.y;
      }
      *dst = __floats2bfloat162_rn(v0, v1);
    }
  }
}

template <int D>
cudaError_t launch_d(const WinParams& p, cudaStream_t s) {
  const size_t smem = (size_t)kRows * D * 2 + 4 * (size_t)kKeys * D * 2 + 1024;
  cudaError_t e = cudaFuncSetAttribute(window_attn_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.T + kRows - 1) / kRows, p.B * p.H);
  window_attn_kernel<D><<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool window_attn_supported(int d, int dv, int dtype) {
  return dtype == TTT_BF16 && d == dv && (d == 64 || d == 128 || d == 256);
}

cudaError_t launch_window_attn(const TokView& q, const TokView& k, const TokView& v,
                               const TokViewMut& out, int B, int H, int T, int d, int window,
                               int accumulate, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  WinParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.B = B;
  p.H = H;
  p.T = T;
  p.window = window;
  p.accumulate = accumulate;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  switch (d) {
    case 64: return launch_d<64>(p, s);
    case 128: return launch_d<128>(p, s);
    case 256: return launch_d<256>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ttt
