// TTT-Linear / inner-product layer forward for bf16 tokens, fp32 fast weights.
//
// The rule (see "Test-Time Training (TTT)" summary, "병렬화: Mini-batch
// Gradient Descent"): per chunk with start weights W_{t'},
//   e_i = k_i W_{t'} - v_i  (MSE)   or   e_i = -v_i  (inner product),
//   W_t = W_{t'} - sum_{i=t'}^{t} eta_i k_i^T e_i,   y_t = q_t W_t.
// Tokens are processed in blocks of 16 that never cross a chunk boundary. With
// W_cur the weights after the previous block (fp32) and, for the block,
// P[t][i] = -eta_i (q_t . k_i) for i <= t (0 otherwise):
//   E^T = W_{t'}^T K^T - V^T               [dv x 16]
//   Y^T = W_cur^T Q^T + E^T P^T            [dv x 16]   (= (Q W_cur - tril(QK^T)N E)^T)
//   W_cur^T += (-E^T N) K                  [dv x dk]
// and at a chunk end W_{t'} <- W_cur. For the inner-product loss E does not
// depend on W, so the chunk size has no effect and blocks of 16 are used.
//
// Layout on the chip: one CTA per (batch, head). Consumer warp w owns dv rows
// [16w, 16w+16) of W^T and keeps them in registers for the whole sequence, as
// the fp32 accumulator fragments of m16n8k16 tensor-core MMAs; the chunk-start
// copy W_{t'}^T is kept as bf16 A-operand fragments. dv columns of W are
// independent under this rule, so warps never exchange state. Accumulator
// fragments convert to A-operand fragments of the next MMA (E^T -> A of the
// update and of E^T P^T) and, transposed, to B-operand fragments (P -> P^T)
// without data movement, so the dependent chain per block stays in registers.
// A producer warp streams Q, K, V blocks with TMA (128-byte swizzle) into a
// ring of shared-memory stages guarded by mbarriers (bounded waits).
#include "common.cuh"
#include "tma.cuh"

namespace ttt {
namespace {

constexpr int kTB = 16;      // tokens per block
constexpr int kStages = 8;   // shared-memory ring depth

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Byte offset of element (row, col) in a [16 x D] bf16 tile stored as D/64
// TMA boxes of [16 x 64] with the 128-byte swizzle (16-byte chunk index XOR
// row % 8). Each box is 2 KB; tiles are 1 KB aligned.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  int box = col >> 6, c = col & 63;
  return box * 2048 + row * 128 + ((((c >> 3) ^ (row & 7))) << 4) + ((c & 7) << 1);
}

template <int D>
struct Smem {
  static constexpr int kTile = kTB * D * 2;  // bytes of one [16 x D] bf16 tile
  alignas(1024) uint8_t q[kStages][kTile];
  alignas(1024) uint8_t k[kStages][kTile];
  alignas(1024) uint8_t v[kStages][kTile];
  float eta[kStages][kTB];
  __nv_bfloat16 ostage[D / 16][kTB][16];  // per-warp output staging [t][r]
  uint64_t full[kStages];
  uint64_t empty[kStages];
};

struct Params {
  CUtensorMap tq, tk, tv;  // 4-d maps {D, T, H, B}, box {64, 16, 1, 1}
  EtaView eta;
  const float* W0;
  int64_t w0_sb;
  TokViewMut out;
  float* W_final;
  int B, H, T, chunk, loss;
  int* status;
};

// Next block [s, s + nb) and whether it ends a chunk.
__device__ __forceinline__ void next_block(const Params& p, int s, int& nb, bool& chunk_end) {
  if (p.loss == TTT_LOSS_MSE) {
    int ce = (int)min((int64_t)(s / p.chunk + 1) * p.chunk, (int64_t)p.T);
    nb = min(kTB, ce - s);
    chunk_end = (s + nb == ce);
  } else {
    nb = min(kTB, p.T - s);
    chunk_end = true;
  }
}

template <int D, int LOSS>
__global__ void __launch_bounds__((D / 16 + 1) * 32, 1)
ttt_linear_bf16_kernel(const __grid_constant__ Params p) {
  constexpr int NW = D / 16;   // consumer warps
  constexpr int NT = D / 8;    // n-tiles of W^T along dk
  constexpr int KB = D / 16;   // k-blocks along dk
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], NW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
    }
    // Learning rates are loaded four blocks ahead into a ring of four register
    // slots (lane l < 16 holds eta of the block's token l). The loop is
    // unrolled by four so every slot keeps a fixed register: a slot is only
    // read when its block is issued, four iterations after its load.
    const float* eta = p.eta.p + b * p.eta.sb + h * p.eta.sh;
    int s_next = 0;  // start of the next block to enter the ring
    auto fill = [&](int& sr, int& nr, float& er) {
      int nb = 0;
      bool ce;
      if (s_next < p.T) next_block(p, s_next, nb, ce);
      sr = s_next;
      nr = nb;
      er = (lane < nb) ? eta[(int64_t)(s_next + lane) * p.eta.st] : 0.f;
      s_next += nb;
    };
    int sr0, sr1, sr2, sr3, nr0, nr1, nr2, nr3;
    float er0, er1, er2, er3;
    fill(sr0, nr0, er0);
    fill(sr1, nr1, er1);
    fill(sr2, nr2, er2);
    fill(sr3, nr3, er3);
    int it = 0;
    // issue one block from a slot, then refill the slot four blocks ahead
    auto issue = [&](int& sr, int& nr, float& er) -> bool {
      if (nr == 0) return false;
      const int st = it % kStages;
      if (it >= kStages && !mbar_wait(&sm.empty[st], ((it / kStages) - 1) & 1, p.status))
        return false;
      if (lane < kTB) sm.eta[st][lane] = er;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.full[st], 3 * Smem<D>::kTile);
        for (int x = 0; x < D / 64; ++x) {
          tma_load_4d(sm.q[st] + x * 2048, &p.tq, &sm.full[st], x * 64, sr, h, b);
          tma_load_4d(sm.k[st] + x * 2048, &p.tk, &sm.full[st], x * 64, sr, h, b);
          tma_load_4d(sm.v[st] + x * 2048, &p.tv, &sm.full[st], x * 64, sr, h, b);
        }
      }
      ++it;
      fill(sr, nr, er);
      return true;
    };
    while (issue(sr0, nr0, er0) && issue(sr1, nr1, er1) && issue(sr2, nr2, er2) &&
           issue(sr3, nr3, er3)) {
    }
    return;
  }

  // ---------------- consumers ----------------
  const int g = lane >> 2, c4 = lane & 3;
  const int r0 = warp * 16;
  const float* W0 = p.W0 + b * p.w0_sb + (int64_t)h * D * D;

  // W_cur^T fragments: Wc[j] covers rows r0+{g, g+8}, cols dk 8j+2c4+{0,1}.
  float Wc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int c = 8 * j + 2 * c4;
    Wc[j][0] = W0[(int64_t)c * D + r0 + g];
    Wc[j][1] = W0[(int64_t)(c + 1) * D + r0 + g];
    Wc[j][2] = W0[(int64_t)c * D + r0 + g + 8];
    Wc[j][3] = W0[(int64_t)(c + 1) * D + r0 + g + 8];
  }
  // Wy: W_cur^T as bf16 A fragments per k-block (operand of W_cur^T Q^T),
  // packed once after every block. Ws: the chunk-start copy W_{t'}^T (MSE).
  uint32_t Wy[KB][4], Ws[KB][4];
  auto pack_cur = [&]() {
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
      Wy[kb][0] = pack_bf16(Wc[2 * kb][0], Wc[2 * kb][1]);
      Wy[kb][1] = pack_bf16(Wc[2 * kb][2], Wc[2 * kb][3]);
      Wy[kb][2] = pack_bf16(Wc[2 * kb + 1][0], Wc[2 * kb + 1][1]);
      Wy[kb][3] = pack_bf16(Wc[2 * kb + 1][2], Wc[2 * kb + 1][3]);
    }
  };
  auto start_chunk = [&]() {
#pragma unroll
    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
      for (int u = 0; u < 4; ++u) Ws[kb][u] = Wy[kb][u];
  };
  pack_cur();
  if constexpr (LOSS == TTT_LOSS_MSE) start_chunk();

  const int mi = lane >> 3, rr = lane & 7;
  int it = 0;
  for (int s = 0; s < p.T; ++it) {
    int nb;
    bool chunk_end;
    next_block(p, s, nb, chunk_end);
    const int st = it % kStages;
    if (!mbar_wait(&sm.full[st], (it / kStages) & 1, p.status)) return;
    const uint32_t qa = smem_u32(sm.q[st]), ka = smem_u32(sm.k[st]);
    const uint8_t* vb = sm.v[st];
    const float* et = sm.eta[st];

    float E[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int t = 8 * nt + 2 * c4;
      auto vv = [&](int tt, int r) {
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vb + sw_off(tt, r)));
      };
      E[nt][0] = -vv(t, r0 + g);
      E[nt][1] = -vv(t + 1, r0 + g);
      E[nt][2] = -vv(t, r0 + g + 8);
      E[nt][3] = -vv(t + 1, r0 + g + 8);
    }
    const int i0 = 2 * c4;
    const float n0 = -et[i0], n1 = -et[i0 + 1], n8 = -et[i0 + 8], n9 = -et[i0 + 9];

    // Three independent products, each split over even / odd k-blocks so that
    // no accumulator chain is longer than KB / 2:
    //   E^T = W_{t'}^T K^T - V^T,  S = Q K^T,  Y^T = W_cur^T Q^T.
    // K and Q enter as B operands (k = dk, n = token), Q also as A (rows token).
    float E2[2][4] = {}, S[2][4] = {}, S2[2][4] = {}, Y[2][4] = {}, Y2[2][4] = {};
#pragma unroll
    for (int kb = 0; kb < KB; kb += 2) {
      uint32_t Bk[2][4], Bq[2][4], Aq[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        ldsm_x4(Bk[u], ka + sw_off(8 * (mi >> 1) + rr, 16 * (kb + u) + 8 * (mi & 1)));
        ldsm_x4(Aq[u], qa + sw_off(rr + 8 * (mi & 1), 16 * (kb + u) + 8 * (mi >> 1)));
        ldsm_x4(Bq[u], qa + sw_off(8 * (mi >> 1) + rr, 16 * (kb + u) + 8 * (mi & 1)));
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        if constexpr (LOSS == TTT_LOSS_MSE) {
          mma16816(E[nt], Ws[kb], Bk[0][2 * nt], Bk[0][2 * nt + 1]);
          mma16816(E2[nt], Ws[kb + 1], Bk[1][2 * nt], Bk[1][2 * nt + 1]);
        }
        mma16816(S[nt], Aq[0], Bk[0][2 * nt], Bk[0][2 * nt + 1]);
        mma16816(S2[nt], Aq[1], Bk[1][2 * nt], Bk[1][2 * nt + 1]);
        mma16816(Y[nt], Wy[kb], Bq[0][2 * nt], Bq[0][2 * nt + 1]);
        mma16816(Y2[nt], Wy[kb + 1], Bq[1][2 * nt], Bq[1][2 * nt + 1]);
      }
    }
    // K^T fragments for the update (issued while the products run)
    uint32_t Kt[NT / 2][4];
#pragma unroll
    for (int j = 0; j < NT; j += 2) ldsm_x4_t(Kt[j / 2], ka + sw_off(rr + 8 * (mi & 1), 8 * (j + (mi >> 1))));

    // P = -eta_i S[t][i] for i <= t, as B fragments of P^T (n-tile = t).
    uint32_t Pb[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int ii = 8 * nt + 2 * c4;
      const float e0 = nt ? n8 : n0, e1 = nt ? n9 : n1;
      const int t0 = g, t1 = g + 8;
      const float s0 = S[nt][0] + S2[nt][0], s1 = S[nt][1] + S2[nt][1];
      const float s2 = S[nt][2] + S2[nt][2], s3 = S[nt][3] + S2[nt][3];
      Pb[0][nt] = pack_bf16((ii <= t0) ? e0 * s0 : 0.f, (ii + 1 <= t0) ? e1 * s1 : 0.f);
      Pb[1][nt] = pack_bf16((ii <= t1) ? e0 * s2 : 0.f, (ii + 1 <= t1) ? e1 * s3 : 0.f);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int u = 0; u < 4; ++u) E[nt][u] += E2[nt][u];

    // W_cur^T += (-E^T N) K   (8 independent MMAs)
    {
      const uint32_t ea[4] = {pack_bf16(n0 * E[0][0], n1 * E[0][1]),
                              pack_bf16(n0 * E[0][2], n1 * E[0][3]),
                              pack_bf16(n8 * E[1][0], n9 * E[1][1]),
                              pack_bf16(n8 * E[1][2], n9 * E[1][3])};
#pragma unroll
      for (int j = 0; j < NT; j += 2) {
        mma16816(Wc[j], ea, Kt[j / 2][0], Kt[j / 2][1]);
        mma16816(Wc[j + 1], ea, Kt[j / 2][2], Kt[j / 2][3]);
      }
    }
    // Y^T += E^T P^T
    {
      const uint32_t ea[4] = {pack_bf16(E[0][0], E[0][1]), pack_bf16(E[0][2], E[0][3]),
                              pack_bf16(E[1][0], E[1][1]), pack_bf16(E[1][2], E[1][3])};
      mma16816(Y[0], ea, Pb[0][0], Pb[0][1]);
      mma16816(Y[1], ea, Pb[1][0], Pb[1][1]);
    }

    // Output: stage Y^T -> [t][r] and store 16 rows x 32 bytes.
    __nv_bfloat16(*os)[16] = sm.ostage[warp];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int t = 8 * nt + 2 * c4;
      os[t][g] = __float2bfloat16_rn(Y[nt][0] + Y2[nt][0]);
      os[t + 1][g] = __float2bfloat16_rn(Y[nt][1] + Y2[nt][1]);
      os[t][g + 8] = __float2bfloat16_rn(Y[nt][2] + Y2[nt][2]);
      os[t + 1][g + 8] = __float2bfloat16_rn(Y[nt][3] + Y2[nt][3]);
    }
    __syncwarp();
    {
      const int t = lane >> 1, half = lane & 1;
      if (t < nb) {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out.p) + b * p.out.sb + h * p.out.sh +
                           (int64_t)(s + t) * p.out.st + r0 + 8 * half;
        *reinterpret_cast<uint4*>(o) = *reinterpret_cast<const uint4*>(&os[t][8 * half]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);
    pack_cur();
    if constexpr (LOSS == TTT_LOSS_MSE)
      if (chunk_end) start_chunk();
    s += nb;
  }

  if (p.W_final) {
    float* Wf = p.W_final + (int64_t)bh * D * D;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int c = 8 * j + 2 * c4;
      Wf[(int64_t)c * D + r0 + g] = Wc[j][0];
      Wf[(int64_t)(c + 1) * D + r0 + g] = Wc[j][1];
      Wf[(int64_t)c * D + r0 + g + 8] = Wc[j][2];
      Wf[(int64_t)(c + 1) * D + r0 + g + 8] = Wc[j][3];
    }
  }
}

bool token_map(CUtensorMap* m, const TokView& v, int B, int H, int T, int D) {
  uint64_t dims[4] = {(uint64_t)D, (uint64_t)T, (uint64_t)H, (uint64_t)B};
  uint64_t strides[3] = {(uint64_t)v.st * 2, (uint64_t)v.sh * 2, (uint64_t)v.sb * 2};
  uint32_t box[4] = {64, kTB, 1, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, v.p, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int D>
cudaError_t launch(const LinearArgs& a, cudaStream_t s) {
  Params p;
  // TMA needs non-zero strides for every dim; a size-1 dim may carry any stride.
  TokView q = a.q, k = a.k, v = a.v;
  for (TokView* x : {&q, &k, &v}) {
    if (a.B == 1) x->sb = (int64_t)a.H * a.T * D;
    if (a.H == 1) x->sh = (int64_t)a.T * D;
    if (a.T == 1) x->st = D;
  }
  if (!token_map(&p.tq, q, a.B, a.H, a.T, D) || !token_map(&p.tk, k, a.B, a.H, a.T, D) ||
      !token_map(&p.tv, v, a.B, a.H, a.T, D))
    return cudaErrorInvalidValue;
  p.eta = a.eta;
  p.W0 = a.W0;
  p.w0_sb = a.w0_sb;
  p.out = a.out;
  p.W_final = a.W_final;
  p.B = a.B;
  p.H = a.H;
  p.T = a.T;
  p.chunk = a.chunk;
  p.loss = a.loss;
  p.status = a.status;
  const size_t smem = sizeof(Smem<D>) + 1024;
  auto kernel = a.loss == TTT_LOSS_MSE ? ttt_linear_bf16_kernel<D, TTT_LOSS_MSE>
                                       : ttt_linear_bf16_kernel<D, TTT_LOSS_NEG_DOT>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kernel<<<a.B * a.H, (D / 16 + 1) * 32, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ttt_linear_bf16(const LinearArgs& a, cudaStream_t s, bool* supported) {
  *supported = true;
  // head sizes without a tensor-core kernel: fp32 arithmetic on the CUDA cores
  if (!((a.dk == a.dv) && (a.dk == 64 || a.dk == 128))) return launch_ttt_linear_cc_bf16(a, s);
  if (la_tc_supported(a)) return launch_la_tc(a, s);
  if (ttt_linear_wy_supported(a)) return launch_ttt_linear_wy(a, s);
  return a.dk == 64 ? launch<64>(a, s) : launch<128>(a, s);
}

}  // namespace ttt
