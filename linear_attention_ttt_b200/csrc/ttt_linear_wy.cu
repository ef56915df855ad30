// TTT-Linear (MSE loss) forward for head dim dk = dv = 64, bf16 tokens, fp32
// fast weights, in groups of 64 tokens (four 16-token sub-blocks).
//
// The rule ("Test-Time Training (TTT)" summary, "병렬화: Mini-batch Gradient
// Descent"): per chunk with start weights W_{t'},
//   e_i = k_i W_{t'} - v_i,   W_t = W_{t'} - sum_{i=t'}^{t} eta_i k_i^T e_i,
//   y_t = q_t W_t.
// Within a group that starts with weights W_g (N_c = diag(eta) of sub-block c):
//   e_i for sub-block c:  E_c = K_c W_{s(c)} - V_c - sum_{c' < c, other chunk}
//                               K_c K_{c'}^T N_{c'} E_{c'}
// where W_{s(c)} is the start of the chunk that is open when the group starts
// (the correction terms rebuild the start weights of chunks that begin inside
// the group, because W at such a start is W_g minus the updates of the earlier
// sub-blocks), and, for every token t of the group,
//   y_t = q_t W_g - sum_{i <= t in group} eta_i (q_t . k_i) e_i,
//   W_{g+1} = W_g - sum_{i in group} eta_i k_i^T e_i.
// These are the same quantities as the chunk-by-chunk recurrence, so the
// sequential dependence per sub-block shrinks to one 16x16 correction MMA
// (block forward substitution), while the products with W, Q K^T and K K^T
// for the whole group are independent and keep the tensor pipe busy.
// Valid when every chunk boundary falls on a group or sub-block boundary and
// the chunk open at each group start starts there or earlier: chunk 16, 32 or
// a multiple of 64.
//
// Layout on the chip: one CTA per (batch, head) with eight consumer warps in
// two roles. Chain warp w (0-3) owns dv rows [16w, 16w+16) of W^T as
// m16n8k16 accumulator fragments (transposed form: E^T, Y^T and W^T have dv
// as their row dimension) and runs the W-dependent chain of a group: E0, the
// forward substitution and the W update. Output warp w + 4 owns the same dv
// rows and forms Y^T from the group-start weights and the chain warp's errors,
// which it receives through shared memory at two pairwise named barriers.
// Two warps per sub-partition let the MMA chains of one hide the latencies of
// the other. The 16 token-block products of the group (10 blocks of Q K^T, 6
// of K K^T) are split over all eight warps and exchanged through shared
// memory already in the B-fragment order every lane reads. The output tile of
// the group is assembled in shared memory and written as 128-byte rows. A
// producer warp streams 64-token Q, K, V tiles with TMA into a 4-stage ring
// (bounded waits).
#include "common.cuh"
#include "tma.cuh"

namespace ttt {
namespace {

constexpr int D = 64;
constexpr int kG = 64;        // tokens per group
constexpr int kSub = 4;       // 16-token sub-blocks per group
constexpr int kStages = 4;
constexpr int kRowBlocks = 4;  // 16 dv rows each
constexpr int kWarps = 2 * kRowBlocks;  // consumer warps: 4 chain + 4 output
constexpr int kThreads = (kWarps + 1) * 32;
// Named barriers (0 is __syncthreads): all consumers; per row block, the
// chain warp's errors and its next group-start weights for the output warp.
constexpr int kBarConsumers = 1;
constexpr int kBarErr = 2;     // + row block
constexpr int kBarW = 6;       // + row block
constexpr int kTile = kG * D * 2;  // one [64 x 64] bf16 tile, 8 KB
constexpr int kProducts = 16;      // 10 Q K^T blocks + 6 K K^T blocks

// Product p = 4w + j: kind (0: S = Q_c K_c'^T, 1: M = K_c K_c'^T), c, c',
// as codes kind << 4 | c << 2 | c', one byte each in two 64-bit literals:
//   S (0,0) (1,0) (1,1) (2,0) (2,1) (2,2) (3,0) (3,1) (3,2) (3,3),
//   M (1,0) (2,0) (2,1) (3,0) (3,1) (3,2).
__host__ __device__ constexpr int prod_code(int kind, int c, int cp) {
  return (kind << 4) | (c << 2) | cp;
}
__host__ __device__ constexpr uint64_t prod_bits(int lo) {
  const int codes[kProducts] = {prod_code(0, 0, 0), prod_code(0, 1, 0), prod_code(0, 1, 1),
                                prod_code(0, 2, 0), prod_code(0, 2, 1), prod_code(0, 2, 2),
                                prod_code(0, 3, 0), prod_code(0, 3, 1), prod_code(0, 3, 2),
                                prod_code(0, 3, 3), prod_code(1, 1, 0), prod_code(1, 2, 0),
                                prod_code(1, 2, 1), prod_code(1, 3, 0), prod_code(1, 3, 1),
                                prod_code(1, 3, 2)};
  uint64_t b = 0;
  for (int i = 0; i < 8; ++i) b |= (uint64_t)codes[lo + i] << (8 * i);
  return b;
}
__device__ __forceinline__ int prod_of(int pi) {
  constexpr uint64_t kLo = prod_bits(0), kHi = prod_bits(8);
  return (int)(((pi < 8 ? kLo : kHi) >> (8 * (pi & 7))) & 0x1f);
}
// Index of S block (c, c') and M block (c, c') in the table.
__host__ __device__ constexpr int s_index(int c, int cp) { return c * (c + 1) / 2 + cp; }
__host__ __device__ constexpr int m_index(int c, int cp) { return 10 + c * (c - 1) / 2 + cp; }

struct Smem {
  alignas(1024) uint8_t q[kStages][kTile];
  alignas(1024) uint8_t k[kStages][kTile];
  alignas(1024) uint8_t v[kStages][kTile];
  alignas(1024) uint8_t ostage[2][kTile];            // output tile [64 t][64 dv]
  uint32_t frag[2][kProducts][2][2][32];             // [buf][product][n-tile][b0|b1][lane]
  uint32_t wy[kRowBlocks][4][4][32];                 // group-start W^T (bf16 A fragments)
  uint32_t ae[2][kRowBlocks][kSub][4][32];           // errors E^T (bf16 A fragments)
  float eta[kStages][kG];
  uint64_t full[kStages], empty[kStages];
  int abort;
};

struct Params {
  CUtensorMap tq, tk, tv;  // {64, T, H, B}, box {64, 64, 1, 1}
  EtaView eta;
  const float* W0;
  int64_t w0_sb;
  TokViewMut out;
  float* W_final;
  int B, H, T, chunk;
  int* status;
};

// Byte offset of element (row, col) of a [64 x 64] bf16 tile with the 128-byte
// swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t sw(int row, int col) {
  return row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + ((col & 7) << 1);
}

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

__global__ void __launch_bounds__(kThreads, 1) ttt_linear_wy_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  if (!TTT_BOUNDS(bh < p.B * p.H, p.status)) return;  // uniform over the CTA
  const int ngroups = (p.T + kG - 1) / kG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kWarps);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
    }
    // Learning rates four groups ahead in four fixed register slots (two per
    // lane per group); the loop is unrolled by four so no slot is moved.
    const float* eta = p.eta.p + b * p.eta.sb + h * p.eta.sh;
    auto load_eta = [&](int j, float& e0, float& e1) {
      const int t = j * kG + lane;
      e0 = (j < ngroups && t < p.T) ? eta[(int64_t)t * p.eta.st] : 0.f;
      e1 = (j < ngroups && t + 32 < p.T) ? eta[(int64_t)(t + 32) * p.eta.st] : 0.f;
    };
    float r0a, r0b, r1a, r1b, r2a, r2b, r3a, r3b;
    load_eta(0, r0a, r0b);
    load_eta(1, r1a, r1b);
    load_eta(2, r2a, r2b);
    load_eta(3, r3a, r3b);
    int j = 0;
    auto issue = [&](float& ea, float& eb) -> bool {
      if (j >= ngroups) return false;
      const int st = j % kStages;
      if (j >= kStages && !mbar_wait(&sm.empty[st], ((j / kStages) - 1) & 1, p.status))
        return false;
      sm.eta[st][lane] = ea;
      sm.eta[st][lane + 32] = eb;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.full[st], 3 * kTile);
        tma_load_4d(sm.q[st], &p.tq, &sm.full[st], 0, j * kG, h, b);
        tma_load_4d(sm.k[st], &p.tk, &sm.full[st], 0, j * kG, h, b);
        tma_load_4d(sm.v[st], &p.tv, &sm.full[st], 0, j * kG, h, b);
      }
      load_eta(j + 4, ea, eb);
      ++j;
      return true;
    };
    while (issue(r0a, r0b) && issue(r1a, r1b) && issue(r2a, r2b) && issue(r3a, r3b)) {
    }
    return;
  }

  // ---------------- consumers ----------------
  const int g = lane >> 2, c4 = lane & 3, mi = lane >> 3, rr = lane & 7;
  const bool chain = warp < kRowBlocks;
  const int rb = warp & (kRowBlocks - 1);
  const int r0 = rb * 16;  // this warp's dv rows
  const int tid = threadIdx.x;
  auto bar_consumers = [] { asm volatile("bar.sync %0, %1;" ::"n"(kBarConsumers), "n"(kWarps * 32) : "memory"); };
  auto pair_arrive = [](int id) { asm volatile("bar.arrive %0, 64;" ::"r"(id) : "memory"); };
  auto pair_sync = [](int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); };

  // W_cur^T fragments (chain warps): Wc[j] covers dv rows r0+{g, g+8}, dk
  // columns 8j+2c4+{0,1}.
  float Wc[8][4];
  // Wy: W_g^T as bf16 A fragments per dk block; Ws: start weights of the open chunk.
  uint32_t Wy[4][4], Ws[4][4];
  auto pack_cur = [&]() {
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      Wy[kb][0] = pack_bf16(Wc[2 * kb][0], Wc[2 * kb][1]);
      Wy[kb][1] = pack_bf16(Wc[2 * kb][2], Wc[2 * kb][3]);
      Wy[kb][2] = pack_bf16(Wc[2 * kb + 1][0], Wc[2 * kb + 1][1]);
      Wy[kb][3] = pack_bf16(Wc[2 * kb + 1][2], Wc[2 * kb + 1][3]);
    }
  };
  auto start_chunk = [&]() {
#pragma unroll
    for (int kb = 0; kb < 4; ++kb)
#pragma unroll
      for (int u = 0; u < 4; ++u) Ws[kb][u] = Wy[kb][u];
  };
  auto publish_w = [&]() {  // chain warp -> output warp: the next group-start weights
#pragma unroll
    for (int kb = 0; kb < 4; ++kb)
#pragma unroll
      for (int u = 0; u < 4; ++u) sm.wy[rb][kb][u][lane] = Wy[kb][u];
    pair_arrive(kBarW + rb);
  };
  if (chain) {
    const float* W0 = p.W0 + b * p.w0_sb + (int64_t)h * D * D;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 8 * j + 2 * c4;
      Wc[j][0] = W0[(int64_t)c * D + r0 + g];
      Wc[j][1] = W0[(int64_t)(c + 1) * D + r0 + g];
      Wc[j][2] = W0[(int64_t)c * D + r0 + g + 8];
      Wc[j][3] = W0[(int64_t)(c + 1) * D + r0 + g + 8];
    }
    pack_cur();
    start_chunk();
    if (ngroups > 0) publish_w();
  }

  __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(p.out.p) + b * p.out.sb + h * p.out.sh;
  // rows of the previous group's staged output: every consumer thread stores 16 bytes
  // of 2 rows after the next barrier
  auto store_rows = [&](int gi) {
    const uint8_t* os = sm.ostage[gi & 1];
    const int cch = tid & 7;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t = (tid >> 3) + 32 * i;
      if (gi * kG + t < p.T && TTT_BOUNDS(t < kG && cch * 8 + 8 <= D, p.status))
        *reinterpret_cast<uint4*>(outp + (int64_t)(gi * kG + t) * p.out.st + cch * 8) =
            *reinterpret_cast<const uint4*>(os + t * 128 + ((cch ^ (t & 7)) << 4));
    }
  };

  for (int gi = 0; gi < ngroups; ++gi) {
    const int st = gi % kStages, fb = gi & 1;
    const int g0 = gi * kG;
    const bool ok = mbar_wait(&sm.full[st], (gi / kStages) & 1, p.status);
    // A timed-out wait ends every consumer warp at the barrier of this group:
    // the first failing group is recorded, and a warp still reading the flag
    // of an earlier group does not see a later group's failure.
    if (!ok) atomicCAS(&sm.abort, 0, gi + 1);
    const uint32_t qa = smem_u32(sm.q[st]), ka = smem_u32(sm.k[st]);
    const uint8_t* vb = sm.v[st];
    const float* et = sm.eta[st];

    // 1) this warp's two token-block products, packed in consumer B order
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int pi = 2 * warp + jj;
      const int code = prod_of(pi);
      const int kind = code >> 4, c = (code >> 2) & 3, cp = code & 3;
      float X[2][4] = {};
      const uint32_t abase = kind == 0 ? qa : ka;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        uint32_t a[4], bk[4];
        ldsm_x4(a, abase + sw(16 * c + rr + 8 * (mi & 1), 16 * kb + 8 * (mi >> 1)));
        ldsm_x4(bk, ka + sw(16 * cp + 8 * (mi >> 1) + rr, 16 * kb + 8 * (mi & 1)));
        mma16816(X[0], a, bk[0], bk[1]);
        mma16816(X[1], a, bk[2], bk[3]);
      }
      // S blocks: P[t][i] = -eta_i (q_t . k_i) for i <= t (mask on the diagonal block)
      if (kind == 0) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int i0 = 8 * nt + 2 * c4;
          const float e0 = -et[16 * cp + i0], e1 = -et[16 * cp + i0 + 1];
          const bool diag = c == cp;
          X[nt][0] = (!diag || i0 <= g) ? e0 * X[nt][0] : 0.f;
          X[nt][1] = (!diag || i0 + 1 <= g) ? e1 * X[nt][1] : 0.f;
          X[nt][2] = (!diag || i0 <= g + 8) ? e0 * X[nt][2] : 0.f;
          X[nt][3] = (!diag || i0 + 1 <= g + 8) ? e1 * X[nt][3] : 0.f;
        }
      }
#pragma unroll
      for (int nn = 0; nn < 2; ++nn)
#pragma unroll
        for (int bb = 0; bb < 2; ++bb)
          sm.frag[fb][pi][nn][bb][lane] = pack_bf16(X[bb][2 * nn], X[bb][2 * nn + 1]);
    }

    if (chain) {
      // 2c) E0^T = W_s^T K^T - V^T for the four sub-blocks
      float E[kSub][2][4];
#pragma unroll
      for (int c = 0; c < kSub; ++c) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int t = 16 * c + 8 * nt + 2 * c4;
          auto vv = [&](int tt, int r) {
            return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vb + sw(tt, r)));
          };
          E[c][nt][0] = -vv(t, r0 + g);
          E[c][nt][1] = -vv(t + 1, r0 + g);
          E[c][nt][2] = -vv(t, r0 + g + 8);
          E[c][nt][3] = -vv(t + 1, r0 + g + 8);
        }
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          uint32_t bk[4];
          ldsm_x4(bk, ka + sw(16 * c + 8 * (mi >> 1) + rr, 16 * kb + 8 * (mi & 1)));
          mma16816(E[c][0], Ws[kb], bk[0], bk[1]);
          mma16816(E[c][1], Ws[kb], bk[2], bk[3]);
        }
      }

      // 3c) the products of all warps are visible; the previous group's
      //     output tile is complete (it is stored now)
      bar_consumers();
      {
        const int ab = *reinterpret_cast<volatile int*>(&sm.abort);
        if (ab != 0 && ab <= gi + 1) return;
      }
      if (gi > 0) store_rows(gi - 1);

      // 4c) forward substitution: E_c -= sum over earlier sub-blocks of other
      //     chunks of (-N E_c')^T (K_c' K_c^T); As[c] = (-N_c E_c)^T as A fragments
      int chunk_id[kSub];
#pragma unroll
      for (int c = 0; c < kSub; ++c) chunk_id[c] = (g0 + 16 * c) / p.chunk;
      uint32_t As[kSub][4];
#pragma unroll
      for (int c = 0; c < kSub; ++c) {
#pragma unroll
        for (int cp = 0; cp < c; ++cp) {
          if (chunk_id[cp] == chunk_id[c]) continue;
          const uint32_t* f = &sm.frag[fb][m_index(c, cp)][0][0][0];
          mma16816(E[c][0], As[cp], f[0 * 64 + 0 * 32 + lane], f[0 * 64 + 1 * 32 + lane]);
          mma16816(E[c][1], As[cp], f[1 * 64 + 0 * 32 + lane], f[1 * 64 + 1 * 32 + lane]);
        }
        const float e0 = -et[16 * c + 2 * c4], e1 = -et[16 * c + 2 * c4 + 1];
        const float e8 = -et[16 * c + 8 + 2 * c4], e9 = -et[16 * c + 9 + 2 * c4];
        As[c][0] = pack_bf16(e0 * E[c][0][0], e1 * E[c][0][1]);
        As[c][1] = pack_bf16(e0 * E[c][0][2], e1 * E[c][0][3]);
        As[c][2] = pack_bf16(e8 * E[c][1][0], e9 * E[c][1][1]);
        As[c][3] = pack_bf16(e8 * E[c][1][2], e9 * E[c][1][3]);
        uint32_t* ae = &sm.ae[fb][rb][c][0][0];
        ae[0 * 32 + lane] = pack_bf16(E[c][0][0], E[c][0][1]);
        ae[1 * 32 + lane] = pack_bf16(E[c][0][2], E[c][0][3]);
        ae[2 * 32 + lane] = pack_bf16(E[c][1][0], E[c][1][1]);
        ae[3 * 32 + lane] = pack_bf16(E[c][1][2], E[c][1][3]);
      }
      pair_arrive(kBarErr + rb);  // errors of this group -> output warp

      // 5c) W_g^T += sum_c (-N_c E_c)^T K_c
#pragma unroll
      for (int c = 0; c < kSub; ++c)
#pragma unroll
        for (int jn = 0; jn < 8; jn += 2) {
          uint32_t r[4];
          ldsm_x4_t(r, ka + sw(16 * c + rr + 8 * (mi & 1), 8 * (jn + (mi >> 1))));
          mma16816(Wc[jn], As[c], r[0], r[1]);
          mma16816(Wc[jn + 1], As[c], r[2], r[3]);
        }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&sm.empty[st]);  // this warp is done with the stage
      pack_cur();
      if ((g0 + kG) % p.chunk == 0) start_chunk();
      if (gi + 1 < ngroups) publish_w();
    } else {
      // 2y) Y0^T = W_g^T Q^T with the group-start weights from the chain warp
      pair_sync(kBarW + rb);
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
#pragma unroll
        for (int u = 0; u < 4; ++u) Wy[kb][u] = sm.wy[rb][kb][u][lane];
      float Y[kSub][2][4];
#pragma unroll
      for (int c = 0; c < kSub; ++c) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int u = 0; u < 4; ++u) Y[c][nt][u] = 0.f;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          uint32_t bq[4];
          ldsm_x4(bq, qa + sw(16 * c + 8 * (mi >> 1) + rr, 16 * kb + 8 * (mi & 1)));
          mma16816(Y[c][0], Wy[kb], bq[0], bq[1]);
          mma16816(Y[c][1], Wy[kb], bq[2], bq[3]);
        }
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&sm.empty[st]);  // Q of this stage is consumed

      // 3y) see 3c
      bar_consumers();
      {
        const int ab = *reinterpret_cast<volatile int*>(&sm.abort);
        if (ab != 0 && ab <= gi + 1) return;
      }
      if (gi > 0) store_rows(gi - 1);

      // 4y) Y^T_c += sum_{c' <= c} E_c'^T P_{c,c'}^T with the chain warp's errors
      pair_sync(kBarErr + rb);
      uint32_t Ae[kSub][4];
#pragma unroll
      for (int c = 0; c < kSub; ++c)
#pragma unroll
        for (int u = 0; u < 4; ++u) Ae[c][u] = sm.ae[fb][rb][c][u][lane];
#pragma unroll
      for (int c = 0; c < kSub; ++c)
#pragma unroll
        for (int cp = 0; cp <= c; ++cp) {
          const uint32_t* f = &sm.frag[fb][s_index(c, cp)][0][0][0];
          mma16816(Y[c][0], Ae[cp], f[0 * 64 + 0 * 32 + lane], f[0 * 64 + 1 * 32 + lane]);
          mma16816(Y[c][1], Ae[cp], f[1 * 64 + 0 * 32 + lane], f[1 * 64 + 1 * 32 + lane]);
        }

      // 5y) Y^T -> staged [t][dv] bf16 tile
      uint8_t* os = sm.ostage[fb];
#pragma unroll
      for (int c = 0; c < kSub; ++c)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int t = 16 * c + 8 * nt + 2 * c4;
          *reinterpret_cast<__nv_bfloat16*>(os + sw(t, r0 + g)) = __float2bfloat16_rn(Y[c][nt][0]);
          *reinterpret_cast<__nv_bfloat16*>(os + sw(t + 1, r0 + g)) = __float2bfloat16_rn(Y[c][nt][1]);
          *reinterpret_cast<__nv_bfloat16*>(os + sw(t, r0 + g + 8)) = __float2bfloat16_rn(Y[c][nt][2]);
          *reinterpret_cast<__nv_bfloat16*>(os + sw(t + 1, r0 + g + 8)) =
              __float2bfloat16_rn(Y[c][nt][3]);
        }
    }
  }
  bar_consumers();
  if (ngroups > 0) store_rows(ngroups - 1);

  if (chain && p.W_final) {
    float* Wf = p.W_final + (int64_t)bh * D * D;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 8 * j + 2 * c4;
      Wf[(int64_t)c * D + r0 + g] = Wc[j][0];
      Wf[(int64_t)(c + 1) * D + r0 + g] = Wc[j][1];
      Wf[(int64_t)c * D + r0 + g + 8] = Wc[j][2];
      Wf[(int64_t)(c + 1) * D + r0 + g + 8] = Wc[j][3];
    }
  }
}

bool token_map(CUtensorMap* m, const TokView& v, int B, int H, int T) {
  TokView x = v;
  if (B == 1) x.sb = (int64_t)H * T * D;
  if (H == 1) x.sh = (int64_t)T * D;
  if (T == 1) x.st = D;
  uint64_t dims[4] = {(uint64_t)D, (uint64_t)T, (uint64_t)H, (uint64_t)B};
  uint64_t strides[3] = {(uint64_t)x.st * 2, (uint64_t)x.sh * 2, (uint64_t)x.sb * 2};
  uint32_t box[4] = {64, kG, 1, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x.p, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool ttt_linear_wy_supported(const LinearArgs& a) {
  return a.loss == TTT_LOSS_MSE && a.dk == D && a.dv == D && a.T > 0 &&
         (a.chunk == 16 || a.chunk == 32 || a.chunk % kG == 0);
}

cudaError_t launch_ttt_linear_wy(const LinearArgs& a, cudaStream_t s) {
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
  p.chunk = a.chunk;
  p.status = a.status;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(ttt_linear_wy_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ttt_linear_wy_kernel<<<a.B * a.H, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ttt
