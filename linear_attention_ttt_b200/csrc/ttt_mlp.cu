// TTT-MLP forward: a two-layer ReLU MLP fast weight under the mini-batch GD
// rule ("Test-Time Training (TTT)" summary, sections "TTT-MLP" and "병렬화:
// Mini-batch Gradient Descent").
//
// f(x) = W2 ReLU(W1 x + b1) + b2 with W1 [dh][dk], b1 [dh], W2 [dv][dh],
// b2 [dv]; per-token loss 1/2 ||f(k) - v||^2. In a chunk with start
// parameters P_s every gradient is taken at P_s, and token t sees
// P_t = P_s - sum_{i<=t} eta_i grad_i(P_s). For key token i, with
// h_i = W1 k_i + b1, a_i = ReLU(h_i), r_i = W2 a_i + b2 - v_i and
// g_i = (W2^T r_i) [h_i > 0] (ReLU derivative 0 at 0), the gradient is
// (g_i k_i^T, g_i, r_i a_i^T, r_i). So for a query token t:
//   z_t = W1_t q_t + b1_t = W1_s q_t + b1_s - sum_{i<=t} eta_i (q_t . k_i + 1) g_i
//   y_t = W2_t a'_t + b2_t = W2_s a'_t + b2_s - sum_{i<=t} eta_i (a'_t . a_i + 1) r_i,
// with a'_t = ReLU(z_t): the dual (attention-like) form of the chunk.
//
// Layout: one CTA of 512 threads per (batch, head), fp32 arithmetic on the
// CUDA cores. A chunk is walked in blocks of 16 tokens with two parameter
// copies: the chunk-start copy P_s, used for the keys' h, a, r, g (and for the
// queries of a chunk's first block), and the running copy, which holds the
// updates of the chunk's earlier blocks and serves the other queries. P_s
// sits in shared memory when it fits beside the block buffers (d 64, hidden
// 256: 132 KB + 85 KB), else in an fp32 workspace (L2-resident) like the
// running copy; with single-block chunks the running copy is never needed.
#include "common.cuh"

namespace ttt {

namespace {

constexpr int kThreads = 512;  // 16 warps: the product loops are latency-bound
constexpr int kTB = 16;
constexpr int kP = kTB + 1;   // padded token stride of the block buffers
constexpr int kB = 8;         // global reads issued together per thread
static_assert(kThreads % kTB == 0, "paired outputs x, x + kThreads share their token");

// floats of the block buffers (before any shared-memory parameter copy)
__host__ __device__ constexpr int64_t mlp_buf_floats(int dk, int dv, int dh) {
  return (int64_t)(2 * dk + dv + 4 * dh) * kP + 2 * kTB * kP + kTB;
}

template <typename T>
__device__ __forceinline__ float ldt(const TokView& v, int b, int h, int64_t t, int c) {
  return to_f32((static_cast<const T*>(v.p) + b * v.sb + h * v.sh + t * v.st)[c]);
}

// kSP: the chunk-start parameters live in shared memory (when they fit beside
// the block buffers); the running copy stays in the workspace.
template <typename T, bool kSP>
__global__ void __launch_bounds__(kThreads, 1) ttt_mlp_kernel(MlpArgs a) {
  extern __shared__ float smem[];
  const int dk = a.dk, dv = a.dv, dh = a.dh;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int tid = threadIdx.x;
  const int64_t nP = (int64_t)dh * dk + dh + (int64_t)dv * dh + dv;

  // workspace: start and running copies of (W1, b1, W2, b2)
  float* ps = a.ws + (int64_t)bh * 2 * nP;
  float* sW1 = kSP ? smem + mlp_buf_floats(dk, dv, dh) : ps;
  float* sb1 = sW1 + (int64_t)dh * dk;
  float* sW2 = sb1 + dh;
  float* sb2 = sW2 + (int64_t)dv * dh;
  float* rW1 = ps + nP;
  float* rb1 = rW1 + (int64_t)dh * dk;
  float* rW2 = rb1 + dh;
  float* rb2 = rW2 + (int64_t)dv * dh;

  // Block buffers, stored transposed with a padded token stride kP, so that
  // the threads of a warp (which differ in the token or in the feature
  // index) touch distinct banks: X(i, c) = X[c * kP + i] for token i.
  float* Qs = smem;                    // [dk][kP]
  float* Ks = Qs + dk * kP;            // [dk][kP]
  float* Vs = Ks + dk * kP;            // [dv][kP]  v, then r
  float* Hs = Vs + dv * kP;            // [dh][kP]  h, then a = ReLU(h)
  float* Gs = Hs + dh * kP;            // [dh][kP]  g
  float* Zs = Gs + dh * kP;            // [dh][kP]  z, then a' = ReLU(z)
  float* Hm = Zs + dh * kP;            // [dh][kP]  1 where h > 0
  float* S1 = Hm + dh * kP;            // [16][kP]  S1[t][i]
  float* S2 = S1 + kTB * kP;           // [16][kP]
  float* et = S2 + kTB * kP;           // [16]

  // initial parameters into both copies
  {
    const float* src[4] = {a.W1 + (int64_t)(a.p_sb[0] ? bh : h) * dh * dk,
                           a.b1 + (int64_t)(a.p_sb[1] ? bh : h) * dh,
                           a.W2 + (int64_t)(a.p_sb[2] ? bh : h) * dv * dh,
                           a.b2 + (int64_t)(a.p_sb[3] ? bh : h) * dv};
    const int64_t len[4] = {(int64_t)dh * dk, dh, (int64_t)dv * dh, dv};
    float* dst[4] = {sW1, sb1, sW2, sb2};
    float* dst2[4] = {rW1, rb1, rW2, rb2};
    for (int m = 0; m < 4; ++m)
      for (int64_t x = tid; x < len[m]; x += kThreads) dst[m][x] = dst2[m][x] = src[m][x];
  }
  __syncthreads();

  const float* eta = a.eta.p + b * a.eta.sb + h * a.eta.sh;
  for (int cs = 0; cs < a.T; cs += a.chunk) {
    const int ce = min(cs + a.chunk, a.T);
    for (int t0 = cs; t0 < ce; t0 += kTB) {
      const int nt = min(kTB, ce - t0);
      // the queries read the running parameters; at a chunk's first block they
      // equal the start copy, which kSP keeps in shared memory
      const bool first = t0 == cs, last = t0 + kTB >= ce;
      const bool from_start = kSP && first;
      const float* zW1 = from_start ? sW1 : rW1;
      const float* zb1 = from_start ? sb1 : rb1;
      const float* zW2 = from_start ? sW2 : rW2;
      const float* zb2 = from_start ? sb2 : rb2;
      for (int x0 = 0; x0 < kTB * dk; x0 += kB * kThreads) {
        float qv[kB], kv[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int x = x0 + tid + u * kThreads, i = x / dk, c = x % dk;
          const bool ok = x < kTB * dk && i < nt;
          qv[u] = ok ? ldt<T>(a.q, b, h, t0 + i, c) : 0.f;
          kv[u] = ok ? ldt<T>(a.k, b, h, t0 + i, c) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int x = x0 + tid + u * kThreads, i = x / dk, c = x % dk;
          if (x < kTB * dk) Qs[c * kP + i] = qv[u], Ks[c * kP + i] = kv[u];
        }
      }
      for (int x0 = 0; x0 < kTB * dv; x0 += kB * kThreads) {
        float vv[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int x = x0 + tid + u * kThreads, i = x / dv, c = x % dv;
          vv[u] = x < kTB * dv && i < nt ? ldt<T>(a.v, b, h, t0 + i, c) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int x = x0 + tid + u * kThreads, i = x / dv, c = x % dv;
          if (x < kTB * dv) Vs[c * kP + i] = vv[u];
        }
      }
      if (tid < kTB) et[tid] = tid < nt ? eta[(int64_t)(t0 + tid) * a.eta.st] : 0.f;
      __syncthreads();
      // h = W1_s k + b1_s, and z0 = W1_run q + b1_run (running: earlier blocks
      // applied). Each thread takes the outputs x and x + kThreads together (the
      // same token i, since kThreads is a multiple of kTB): four sums side by
      // side, each in its own fixed order, sharing the token loads.
      for (int x = tid; x < kTB * dh; x += 2 * kThreads) {
        const bool two = x + kThreads < kTB * dh;
        const int j = x / kTB, i = x % kTB, j2 = two ? (x + kThreads) / kTB : j;
        float hk = sb1[j], zq = zb1[j], hk2 = sb1[j2], zq2 = zb1[j2];
        const float* w = sW1 + (int64_t)j * dk;
        const float* wr = zW1 + (int64_t)j * dk;
        const float* w2 = sW1 + (int64_t)j2 * dk;
        const float* wr2 = zW1 + (int64_t)j2 * dk;
#pragma unroll 4
        for (int r = 0; r < dk; ++r) {
          const float kr = Ks[r * kP + i], qr = Qs[r * kP + i];
          hk = fmaf(w[r], kr, hk);
          zq = fmaf(wr[r], qr, zq);
          hk2 = fmaf(w2[r], kr, hk2);
          zq2 = fmaf(wr2[r], qr, zq2);
        }
        Hs[j * kP + i] = fmaxf(hk, 0.f);
        Hm[j * kP + i] = hk > 0.f ? 1.f : 0.f;
        Zs[j * kP + i] = zq;
        if (two) {
          Hs[j2 * kP + i] = fmaxf(hk2, 0.f);
          Hm[j2 * kP + i] = hk2 > 0.f ? 1.f : 0.f;
          Zs[j2 * kP + i] = zq2;
        }
      }
      // S1[t][i] = q_t . k_i + 1 (i <= t)
      if (tid < kTB * kTB) {
        const int t = tid / kTB, i = tid % kTB;
        float sv = 0.f;
        if (i <= t) {
          sv = 1.f;
          for (int r = 0; r < dk; ++r) sv = fmaf(Qs[r * kP + t], Ks[r * kP + i], sv);
        }
        S1[t * kP + i] = sv;
      }
      __syncthreads();
      // r = W2_s a + b2_s - v (outputs x and x + kThreads together, as above)
      for (int x = tid; x < kTB * dv; x += 2 * kThreads) {
        const bool two = x + kThreads < kTB * dv;
        const int c = x / kTB, i = x % kTB, c2 = two ? (x + kThreads) / kTB : c;
        float sv = sb2[c], sv2 = sb2[c2];
        const float* w = sW2 + (int64_t)c * dh;
        const float* w2 = sW2 + (int64_t)c2 * dh;
#pragma unroll 4
        for (int j = 0; j < dh; ++j) {
          const float hj = Hs[j * kP + i];
          sv = fmaf(w[j], hj, sv);
          sv2 = fmaf(w2[j], hj, sv2);
        }
        Vs[c * kP + i] = sv - Vs[c * kP + i];
        if (two) Vs[c2 * kP + i] = sv2 - Vs[c2 * kP + i];
      }
      __syncthreads();
      // g = (W2_s^T r) [h > 0] (outputs x and x + kThreads together)
      for (int x = tid; x < kTB * dh; x += 2 * kThreads) {
        const bool two = x + kThreads < kTB * dh;
        const int j = x / kTB, i = x % kTB, j2 = two ? (x + kThreads) / kTB : j;
        float sv = 0.f, sv2 = 0.f;
#pragma unroll 4
        for (int c = 0; c < dv; ++c) {
          const float rc = Vs[c * kP + i];
          sv = fmaf(sW2[(int64_t)c * dh + j], rc, sv);
          sv2 = fmaf(sW2[(int64_t)c * dh + j2], rc, sv2);
        }
        Gs[j * kP + i] = sv * Hm[j * kP + i];
        if (two) Gs[j2 * kP + i] = sv2 * Hm[j2 * kP + i];
      }
      __syncthreads();
      // z = z0 - sum_{i<=t} eta_i S1[t][i] g_i ; a' = ReLU(z)
      for (int x = tid; x < kTB * dh; x += kThreads) {
        const int t = x / dh, j = x % dh;
        float z = Zs[j * kP + t];
        for (int i = 0; i <= t; ++i) z = fmaf(-et[i] * S1[t * kP + i], Gs[j * kP + i], z);
        Zs[j * kP + t] = fmaxf(z, 0.f);
      }
      __syncthreads();
      // S2[t][i] = a'_t . a_i + 1 (i <= t)
      if (tid < kTB * kTB) {
        const int t = tid / kTB, i = tid % kTB;
        float sv = 0.f;
        if (i <= t) {
          sv = 1.f;
          for (int j = 0; j < dh; ++j) sv = fmaf(Zs[j * kP + t], Hs[j * kP + i], sv);
        }
        S2[t * kP + i] = sv;
      }
      __syncthreads();
      // y = W2_run a' + b2_run - sum_{i<=t} eta_i S2[t][i] r_i
      // (outputs x and x + kThreads together: the same token t)
      for (int x = tid; x < kTB * dv; x += 2 * kThreads) {
        const bool two = x + kThreads < kTB * dv;
        const int c = x / kTB, t = x % kTB, c2 = two ? (x + kThreads) / kTB : c;
        if (t < nt) {
          float y = zb2[c], y2 = zb2[c2];
          const float* w = zW2 + (int64_t)c * dh;
          const float* w2 = zW2 + (int64_t)c2 * dh;
#pragma unroll 4
          for (int j = 0; j < dh; ++j) {
            const float zj = Zs[j * kP + t];
            y = fmaf(w[j], zj, y);
            y2 = fmaf(w2[j], zj, y2);
          }
          for (int i = 0; i <= t; ++i) {
            const float sti = -et[i] * S2[t * kP + i];
            y = fmaf(sti, Vs[c * kP + i], y);
            y2 = fmaf(sti, Vs[c2 * kP + i], y2);
          }
          T* o = static_cast<T*>(a.out.p) + b * a.out.sb + h * a.out.sh + (int64_t)(t0 + t) * a.out.st;
          o[c] = T(y);
          if (two) o[c2] = T(y2);
        }
      }
      __syncthreads();
      // running parameters: subtract this block's eta-weighted gradients
      // (the weight updates read and write the workspace in batches of kB
      // elements per thread, so that each batch waits for one L2 round trip).
      // kSP: at a chunk's first block the running values are the start copy in
      // shared memory, and the last block's result, the next start, goes there;
      // the workspace copy is kept only between the blocks of one chunk.
      const bool run_in = kSP && first, run_out = !kSP || !last;
      auto put = [&](float* rp, float* sp, int64_t x, float val) {
        if (run_out) rp[x] = val;
        if (kSP && last) sp[x] = val;
      };
      for (int64_t x0 = 0; x0 < (int64_t)dh * dk; x0 += kB * kThreads) {
        float old[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int64_t x = x0 + tid + u * kThreads;
          old[u] = x < (int64_t)dh * dk ? (run_in ? sW1[x] : rW1[x]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int64_t x = x0 + tid + u * kThreads;
          if (x >= (int64_t)dh * dk) continue;
          const int j = (int)(x / dk), r = (int)(x % dk);
          float sv = 0.f;
          for (int i = 0; i < nt; ++i) sv = fmaf(et[i] * Gs[j * kP + i], Ks[r * kP + i], sv);
          put(rW1, sW1, x, old[u] - sv);
        }
      }
      for (int j = tid; j < dh; j += kThreads) {
        float sv = 0.f;
        for (int i = 0; i < nt; ++i) sv = fmaf(et[i], Gs[j * kP + i], sv);
        put(rb1, sb1, j, (run_in ? sb1[j] : rb1[j]) - sv);
      }
      for (int64_t x0 = 0; x0 < (int64_t)dv * dh; x0 += kB * kThreads) {
        float old[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int64_t x = x0 + tid + u * kThreads;
          old[u] = x < (int64_t)dv * dh ? (run_in ? sW2[x] : rW2[x]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int64_t x = x0 + tid + u * kThreads;
          if (x >= (int64_t)dv * dh) continue;
          const int c = (int)(x / dh), j = (int)(x % dh);
          float sv = 0.f;
          for (int i = 0; i < nt; ++i) sv = fmaf(et[i] * Vs[c * kP + i], Hs[j * kP + i], sv);
          put(rW2, sW2, x, old[u] - sv);
        }
      }
      for (int c = tid; c < dv; c += kThreads) {
        float sv = 0.f;
        for (int i = 0; i < nt; ++i) sv = fmaf(et[i], Vs[c * kP + i], sv);
        put(rb2, sb2, c, (run_in ? sb2[c] : rb2[c]) - sv);
      }
      __syncthreads();
    }
    // chunk end: the running parameters start the next chunk (kSP: the last
    // block's update already wrote them into shared memory)
    for (int64_t x0 = 0; x0 < (kSP ? 0 : nP); x0 += kB * kThreads) {
      float v[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int64_t x = x0 + tid + u * kThreads;
        v[u] = x < nP ? ps[nP + x] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int64_t x = x0 + tid + u * kThreads;
        if (x < nP) ps[x] = v[u];
      }
    }
    __syncthreads();
  }

  float* fin[4] = {a.W1_final, a.b1_final, a.W2_final, a.b2_final};
  const int64_t len[4] = {(int64_t)dh * dk, dh, (int64_t)dv * dh, dv};
  // kSP: the final parameters are the start copy the last block wrote
  const float* run[4] = {kSP ? sW1 : rW1, kSP ? sb1 : rb1, kSP ? sW2 : rW2, kSP ? sb2 : rb2};
  for (int m = 0; m < 4; ++m)
    if (fin[m])
      for (int64_t x = tid; x < len[m]; x += kThreads) fin[m][(int64_t)bh * len[m] + x] = run[m][x];
}

}  // namespace

bool ttt_mlp_supported(int dk, int dv, int dh) { return dk <= 256 && dv <= 256 && dh <= 512; }

size_t ttt_mlp_workspace(const MlpArgs& a) {
  const int64_t nP = (int64_t)a.dh * a.dk + a.dh + (int64_t)a.dv * a.dh + a.dv;
  return (size_t)a.B * a.H * 2 * nP * sizeof(float);
}

cudaError_t launch_ttt_mlp(const MlpArgs& a, bool bf16, cudaStream_t s) {
  const int64_t nP = (int64_t)a.dh * a.dk + a.dh + (int64_t)a.dv * a.dh + a.dv;
  const size_t buf = sizeof(float) * mlp_buf_floats(a.dk, a.dv, a.dh);
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const bool sp = buf + sizeof(float) * nP <= (size_t)optin;
  const size_t smem = buf + (sp ? sizeof(float) * nP : 0);
  auto go = [&](auto kern) {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (r == cudaSuccess) kern<<<a.B * a.H, kThreads, smem, s>>>(a);
    return r;
  };
  if (bf16)
    e = sp ? go(ttt_mlp_kernel<__nv_bfloat16, true>) : go(ttt_mlp_kernel<__nv_bfloat16, false>);
  else
    e = sp ? go(ttt_mlp_kernel<float, true>) : go(ttt_mlp_kernel<float, false>);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace ttt
