/*
 * ttt.h - C ABI of libttt_b200.so: forward pass of chunked test-time-training
 * (TTT) layers with key->value binding, on one NVIDIA B200 (sm_100a).
 *
 * Three operations, each a per-(batch, head) scan over chunks of `chunk`
 * tokens with fast weights W kept in fp32:
 *
 *  ttt_linear_fwd, loss = TTT_LOSS_MSE  (TTT-Linear, mini-batch GD)
 *    "Test-Time Training (TTT)" summary, sections "TTT 정의", "예시 2: DeltaNet
 *    유도", "TTT-Linear" and "병렬화: Mini-batch Gradient Descent": with
 *    t' = t - (t mod chunk),
 *      W_t = W_{t'} - sum_{i=t'}^{t} eta_i k_i^T (k_i W_{t'} - v_i),
 *      y_t = q_t W_t          (row vectors; W is dk x dv).
 *    Equivalently, per chunk (Q, K, V the chunk's rows, N = diag(eta),
 *    tril keeps i <= t): Y = QW - tril(QK^T) N (KW - V);
 *    W <- W - K^T N (KW - V).
 *
 *  ttt_linear_fwd, loss = TTT_LOSS_NEG_DOT  (inner-product loss)
 *    Same page, sections "Linear Attention" and "예시 1: Linear Attention
 *    유도": the gradient -k^T v does not depend on W, so the layer is causal
 *    linear attention with per-token weights: S_t = S_{t-1} + eta_t k_t^T v_t,
 *    y_t = q_t S_t, S_0 = W0; the result does not depend on `chunk`.
 *    ("Test-Time Training with KV Binding Is Secretly Linear Attention",
 *    abstract: TTT with KV binding as a learned linear-attention operator.)
 *
 *  lact_swiglu_fwd  (LaCT large-chunk SwiGLU fast weights)
 *    "Test-Time Training Done Right" review, sections 3.2, 3.3 and 4 /
 *    Figure 3: f(x) = W2 (silu(W1 x) * W3 x); per chunk c the loss
 *    sum_i eta_i * (-f(k_i) . v_i) is differentiated at the current weights,
 *    the gradients G1, G2, G3 are optionally orthogonalised by 5 Newton-Schulz
 *    steps X <- aX + b(XX^T)X + c(XX^T)^2 X, (a,b,c) = (3.4445, -4.7750,
 *    2.0315), from X0 = G / (||G||_F + 1e-7) (Muon), then W <- W - G and every
 *    row of W1, W3 (over dk) and of W2 (over dh) is rescaled to the L2 norm it
 *    had in the initial weights. causal=1: chunk c's queries see the weights
 *    before chunk c's update (apply, then update); causal=0: update with
 *    chunk c, then apply to chunk c.
 *
 * Conventions shared by every entry point
 *  - Tensors are described by ttt_tensor: a device pointer, an element type,
 *    and shape/stride in ELEMENTS (not bytes). Token tensors q, k, v, out are
 *    4-d [B, H, T, d] with any strides whose last one is 1; eta is 3-d
 *    [B, H, T] fp32 with any strides. Weight tensors are contiguous
 *    (row-major) with the shapes given below.
 *  - Alignment: every base pointer must be 16-byte aligned and every stride of
 *    q, k, v, out times the element size must be a multiple of 16 bytes.
 *  - Ownership: all memory is the caller's. The library keeps no pointer past
 *    the call and never frees caller memory. Inputs are read-only; `out` and
 *    the *_final tensors must not overlap any input.
 *  - Asynchrony: work is enqueued on `stream` (a cudaStream_t passed as
 *    void*; NULL = the legacy default stream) and the call returns without
 *    waiting for it. Argument errors are detected on the host before anything
 *    is launched and returned synchronously; nothing is written then.
 *  - Device-side errors: kernels that wait on a barrier give up after a
 *    bounded number of polls and record TTT_ERR_TIMEOUT in a device status
 *    word instead of hanging; ttt_get_device_status() reads and clears it.
 *  - Device state: the status word, the LaCT scratch pool and the
 *    no-allocation array are set up once per device and kept for the life of
 *    the process. Resetting the device (cudaDeviceReset) or tearing down its
 *    primary context invalidates them; calling the library afterwards in the
 *    same process is not supported.
 *  - Supported sizes: B, H, T >= 1 (T = 0 is accepted and does nothing
 *    except copying W0 to W_final); chunk >= 1 (a shorter last chunk is
 *    allowed). TTT-Linear: dk, dv in [1, 256] (bf16: multiples of 8, from
 *    the stride rule); dk = dv = 64 or 128 run the tensor-core kernels, every
 *    other size (dk != dv included) a CUDA-core kernel with fp32
 *    arithmetic. LaCT: d = dk = dv in {64, 128, 256} and dh a multiple of
 *    128 up to 1024, bf16 tokens. Other sizes return TTT_ERR_UNSUPPORTED, and
 *    so do T > 2^30 tokens and B*H > 2^24 (the kernels index tokens and
 *    (batch, head) pairs with 32-bit integers).
 */
#ifndef TTT_B200_H
#define TTT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_OK = 0,
  TTT_ERR_NULL = -1,        /* a required pointer is NULL */
  TTT_ERR_SHAPE = -2,       /* sizes inconsistent across tensors, or ndim wrong */
  TTT_ERR_DTYPE = -3,       /* element type not allowed for this tensor */
  TTT_ERR_LAYOUT = -4,      /* stride or 16-byte alignment rule broken */
  TTT_ERR_UNSUPPORTED = -5, /* valid request the library has no kernel for */
  TTT_ERR_CUDA = -6,        /* a CUDA runtime call failed (launch, memory) */
  TTT_ERR_TIMEOUT = -7,     /* a device-side bounded wait gave up */
  TTT_ERR_ALLOC = -8,       /* stream-ordered scratch allocation failed */
  TTT_ERR_ARG = -9,         /* scalar argument out of range (chunk, enums) */
  TTT_ERR_SCRATCH = -10,    /* scratch need exceeds lact_swiglu_fwd_noalloc's fixed pool */
  TTT_ERR_BOUNDS = -11      /* debug-bounds build only: a kernel index check failed (the
                               access was skipped); reported by ttt_get_device_status */
} ttt_status;

typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;

typedef enum { TTT_LOSS_MSE = 0, TTT_LOSS_NEG_DOT = 1 } ttt_loss;

typedef enum { LACT_UPDATE_GD = 0, LACT_UPDATE_MUON = 1 } lact_update_rule;

/* Gradient exchange of lact_swiglu_fwd_cp: must enqueue on `stream` an
 * in-place sum over all ranks of the n fp32 values at `grads` (device
 * memory), and return 0 (anything else aborts the call with TTT_ERR_CUDA). */
typedef int32_t (*lact_grad_reduce_fn)(float* grads, size_t n, void* stream, void* user);

typedef struct {
  void* data;          /* device pointer, 16-byte aligned */
  int32_t dtype;       /* ttt_dtype */
  int32_t ndim;        /* number of valid entries in shape/stride */
  int64_t shape[4];
  int64_t stride[4];   /* in elements */
} ttt_tensor;

/*
 * TTT-Linear / inner-product layer forward.
 *  q, k   [B,H,T,dk]  fp32 or bf16 (same type for q, k, v, out)
 *  v      [B,H,T,dv]
 *  eta    [B,H,T]     fp32, per-token learning rate
 *  W0     [H,dk,dv] (shared over the batch) or [B,H,dk,dv], fp32, contiguous
 *  chunk  mini-batch size b >= 1
 *  loss   TTT_LOSS_MSE or TTT_LOSS_NEG_DOT
 *  out    [B,H,T,dv]  same type as q
 *  W_final NULL, or [B,H,dk,dv] fp32 contiguous: weights after the last token
 */
ttt_status ttt_linear_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                          const ttt_tensor* eta, const ttt_tensor* W0, int32_t chunk,
                          int32_t loss, const ttt_tensor* out, const ttt_tensor* W_final,
                          void* stream);

/*
 * TTT-Linear / inner-product layer backward (training): the gradients of a
 * scalar objective through ttt_linear_fwd, given dL/dy and dL/dW_final.
 * Same page and sections as ttt_linear_fwd; differentiating the mini-batch
 * rule token by token, with U_t = q_t^T dy_t and R_t = G + sum of U over the
 * tokens t..end of t's chunk (G = dL/dW at the chunk end):
 *   dq_t = dy_t W_t^T,  deta_t = -<R_t, g_t>,
 *   MSE (g_t = k_t^T e_t, e_t = k_t W_s - v_t): de_t = -eta_t k_t R_t,
 *     dk_t = -eta_t R_t e_t^T + de_t W_s^T, dv_t = -de_t,
 *     dL/dW_s = R_s + sum_t k_t^T de_t;
 *   inner product (g_t = -k_t^T v_t): dk_t = eta_t R_t v_t^T,
 *     dv_t = eta_t k_t R_t, dL/dW_s = R_s;
 * dL/dW_s of a chunk is G of the chunk before it; that of the first chunk is
 * dL/dW0.
 *  q, k, v, eta, W0, chunk, loss   as in ttt_linear_fwd
 *  dy       [B,H,T,dv]  same type as q
 *  dW_final NULL (zero) or [B,H,dk,dv] fp32 contiguous
 *  dq, dk   [B,H,T,dk], dv [B,H,T,dv]: same type as q
 *  deta     [B,H,T] fp32 contiguous
 *  dW0      W0's shape, fp32 contiguous; for a W0 shared over the batch
 *           ([H,dk,dv]) the gradient is summed over the batch
 * dk, dv <= 128 (TTT_ERR_UNSUPPORTED otherwise). Arithmetic is fp32 on the
 * CUDA cores, one CTA per (batch, head). The MSE path keeps the start
 * weights of every chunk in a stream-ordered workspace of
 * B*H*ceil(T/chunk)*dk*dv*4 bytes (plus B*H*dk*dv*4 for a shared W0) from
 * the library's pool; failure -> TTT_ERR_ALLOC.
 */
ttt_status ttt_linear_bwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                          const ttt_tensor* eta, const ttt_tensor* W0, int32_t chunk,
                          int32_t loss, const ttt_tensor* dy, const ttt_tensor* dW_final,
                          const ttt_tensor* dq, const ttt_tensor* dk, const ttt_tensor* dv,
                          const ttt_tensor* deta, const ttt_tensor* dW0, void* stream);

/*
 * TTT-MLP layer forward: a two-layer ReLU MLP fast weight,
 *   f(x) = W2 ReLU(W1 x + b1) + b2,
 * trained per chunk by the mini-batch rule of ttt_linear_fwd on the loss
 * 1/2 ||f(k_i) - v_i||^2 ("Test-Time Training (TTT)" summary, sections
 * "TTT-MLP" and "병렬화: Mini-batch Gradient Descent"): all four parameters
 * are fast weights, every gradient of a chunk is taken at the chunk-start
 * parameters, token t's query sees the updates of tokens <= t of its chunk,
 * and the ReLU derivative at 0 is taken as 0.
 *  q, k [B,H,T,dk], v, out [B,H,T,dv]: fp32 or bf16 (one type for all four)
 *  eta  [B,H,T] fp32
 *  W1 [H,dh,dk], b1 [H,dh], W2 [H,dv,dh], b2 [H,dv] (shared over the batch)
 *     or with a leading B (per sequence); fp32 contiguous, read-only
 *  *_final NULL or [B,H,...] fp32 contiguous: parameters after the last token
 * dk, dv <= 256 and dh <= 512 (TTT_ERR_UNSUPPORTED otherwise). Arithmetic is
 * fp32 on the CUDA cores, one CTA per (batch, head), with a stream-ordered
 * workspace of 2 copies of the parameters per (batch, head) from the
 * library's pool (failure -> TTT_ERR_ALLOC).
 */
ttt_status ttt_mlp_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                       const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* b1,
                       const ttt_tensor* W2, const ttt_tensor* b2, int32_t chunk,
                       const ttt_tensor* out, const ttt_tensor* W1_final,
                       const ttt_tensor* b1_final, const ttt_tensor* W2_final,
                       const ttt_tensor* b2_final, void* stream);

/*
 * LaCT SwiGLU layer forward.
 *  q, k [B,H,T,dk], v, out [B,H,T,dv], bf16 with dk == dv (fp32 tokens
 *       return TTT_ERR_UNSUPPORTED)
 *  eta  [B,H,T] fp32
 *  W1, W3 [H,dh,dk] or [B,H,dh,dk]; W2 [H,dv,dh] or [B,H,dv,dh]; fp32,
 *         contiguous, read-only (the scan works on private copies)
 *  chunk  >= 1; update_rule LACT_UPDATE_GD or LACT_UPDATE_MUON; causal 0/1
 * Scratch is taken stream-ordered (cudaMallocFromPoolAsync / cudaFreeAsync on
 * `stream`) from a memory pool the library creates per device and keeps for
 * the process lifetime, so repeated calls reuse the same mapped memory; the
 * device's default pool is not touched. Failure -> TTT_ERR_ALLOC.
 */
ttt_status lact_swiglu_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                           const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                           const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                           int32_t causal, const ttt_tensor* out, void* stream);

/* As lact_swiglu_fwd, also writing the final fast weights (each NULLable):
 * W1_final, W3_final [B,H,dh,dk], W2_final [B,H,dv,dh], fp32 contiguous. */
ttt_status lact_swiglu_fwd_ex(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                              const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                              const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                              int32_t causal, const ttt_tensor* out,
                              const ttt_tensor* W1_final, const ttt_tensor* W2_final,
                              const ttt_tensor* W3_final, void* stream);

/*
 * LaCT SwiGLU layer forward with the momentum update rule.
 *  "Test-Time Training Done Right" review, section 3.3, lists GD, momentum
 *  and Muon as the compared fast-weight update rules and prints no formula
 *  for momentum. This library takes heavy-ball momentum on each matrix's
 *  eta-weighted chunk gradient G (the gradient of lact_swiglu_fwd):
 *      M <- beta * M + G,    W <- W - M,    then the row renorm,
 *  with M = M0 before the first chunk (zero when M?_0 is NULL). beta = 0 is
 *  plain GD. Apply/update order, precision (bf16 operands, fp32 state) and
 *  every other argument are those of lact_swiglu_fwd_ex with update_rule =
 *  LACT_UPDATE_GD.
 *  beta   any finite float (NaN or infinite -> TTT_ERR_ARG)
 *  M1_0, M3_0 [H,dh,dk] or [B,H,dh,dk]; M2_0 [H,dv,dh] or [B,H,dv,dh]; fp32
 *         contiguous, NULLable (zero initial momentum)
 *  M1_final, M3_final [B,H,dh,dk], M2_final [B,H,dv,dh]: fp32 contiguous,
 *         NULLable; the momentum after the last chunk (pass it back as M?_0,
 *         with the *_final weights as W?, to resume on a chunk boundary)
 * Scratch as for lact_swiglu_fwd, plus one fp32 momentum matrix per weight.
 */
ttt_status lact_swiglu_fwd_momentum(const ttt_tensor* q, const ttt_tensor* k,
                                    const ttt_tensor* v, const ttt_tensor* eta,
                                    const ttt_tensor* W1, const ttt_tensor* W2,
                                    const ttt_tensor* W3, int32_t chunk, float beta,
                                    int32_t causal, const ttt_tensor* M1_0,
                                    const ttt_tensor* M2_0, const ttt_tensor* M3_0,
                                    const ttt_tensor* out, const ttt_tensor* W1_final,
                                    const ttt_tensor* W2_final, const ttt_tensor* W3_final,
                                    const ttt_tensor* M1_final, const ttt_tensor* M2_final,
                                    const ttt_tensor* M3_final, void* stream);

/*
 * Context-parallel LaCT forward ("Test-Time Training Done Right" review,
 * section 8: the tokens of a large chunk are split over devices, each
 * computes the update gradient of its share, and the shares are summed).
 * Each rank passes its own token shard: for a global chunk of C tokens
 * split over R ranks, rank r holds sub-block r (C/R tokens) of every chunk,
 * so its q, k, v, eta, out are [B,H,T/R,d] and `chunk` is C/R. The chunk
 * loop is that of lact_swiglu_fwd_ex; after each chunk's gradient GEMMs the
 * library calls `reduce` (on the calling host thread, in chunk order) to
 * sum the gradients over the ranks before Newton-Schulz, the step and the
 * renorm, which every rank then runs on identical data, so the weights stay
 * identical across ranks. `reduce` NULL means one rank (no exchange).
 * Every rank must make the same sequence of calls with the same B, H,
 * chunk count, d, dh and update rule. Scratch as lact_swiglu_fwd.
 */
ttt_status lact_swiglu_fwd_cp(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                              const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                              const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                              int32_t causal, const ttt_tensor* out,
                              const ttt_tensor* W1_final, const ttt_tensor* W2_final,
                              const ttt_tensor* W3_final, lact_grad_reduce_fn reduce,
                              void* reduce_user, void* stream);

/*
 * LaCT SwiGLU layer backward (training): the gradients of a scalar objective
 * through lact_swiglu_fwd_ex, given dL/dy and optionally dL/d(final weights).
 * Same review and sections as lact_swiglu_fwd. The chunks are walked in
 * reverse; each one differentiates, in this order, the row renorm to the
 * initial norms (whose target norms pass gradient back to the initial
 * weights), the step, Newton-Schulz under Muon (through its five polynomial
 * iterations and the Frobenius normalisation), the gradient formulas
 * themselves (second order: through silu, silu' and silu'' of K W1^T), and
 * the SwiGLU apply of the chunk's queries.
 *  q, k, v, eta, W1, W2, W3, chunk, update_rule, causal   as lact_swiglu_fwd
 *           (bf16 or fp32 tokens; d, dh <= 256, 1024; B*H <= 65535)
 *  dy       [B,H,T,dv], same type as q
 *  dW?_final NULL (zero) or [B,H,...] fp32 contiguous
 *  dq, dk   [B,H,T,dk], dv [B,H,T,dv]: same type as q
 *  deta     [B,H,T] fp32 contiguous
 *  dW1, dW2, dW3  the shapes of W1, W2, W3, fp32 contiguous; per-head
 *           weights ([H,...], shared over the batch) get the batch sum
 * Arithmetic: fp32 throughout (batched fp32 GEMMs on the CUDA cores), from a
 * forward recomputed in fp32, so the result is the derivative of the fp32
 * forward. Workspace is stream-ordered from the library's pool (failure ->
 * TTT_ERR_ALLOC).
 */
ttt_status lact_swiglu_bwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                           const ttt_tensor* eta, const ttt_tensor* W1, const ttt_tensor* W2,
                           const ttt_tensor* W3, int32_t chunk, int32_t update_rule,
                           int32_t causal, const ttt_tensor* dy, const ttt_tensor* dW1_final,
                           const ttt_tensor* dW2_final, const ttt_tensor* dW3_final,
                           const ttt_tensor* dq, const ttt_tensor* dk, const ttt_tensor* dv,
                           const ttt_tensor* deta, const ttt_tensor* dW1, const ttt_tensor* dW2,
                           const ttt_tensor* dW3, void* stream);

/*
 * lact_swiglu_fwd_ex without any device memory allocation. (The pages have
 * no counterpart to this call: it exists for callers that cannot allocate.)
 *
 * Who needs it: callers whose device memory is reserved up front by their
 * own allocator (a serving engine or training framework that claims nearly
 * the whole GPU), where a stream-ordered allocation by this library would
 * fail or fragment memory, and latency-critical code that must not contain
 * allocation calls. Arguments, results and errors are those of
 * lact_swiglu_fwd_ex; the caller still passes every input and output.
 *
 * Scratch: a fixed 32 MiB device array inside the library (each device that
 * loads the library holds it until the process exits). A problem whose
 * scratch need exceeds it is rejected with TTT_ERR_SCRATCH before anything
 * is launched. The need per (batch, head), with E = 2*dh*dk + dv*dh weight
 * elements, R = 2*dh + dv weight rows and c = min(chunk, T), is
 *   4 bytes x (2*E + R)  +  2 bytes x (E + 4*c*dh) x (2 under Muon),
 * plus, under Muon when the gradients are not 128 x 512 (dk = dv = 128 and
 * dh = 512 keep Newton-Schulz on chip), 4 bytes x 3 x (16*s*s + dh*dk + 64)
 * with s = min(dk, dh); the sum over all (batch, head) pairs gets 4096
 * bytes of alignment slack. Example: dk = dv = 128, dh = 512, chunk 1024,
 * GD: 1,577,472 + 4,587,520 = 6,164,992 bytes per (batch, head), so up to
 * five (batch, head) pairs fit.
 * The first call on a device looks up the array's device address with that
 * device current and keeps it for the life of the process; make that first
 * call before any stream capture. A cudaDeviceReset (or any teardown of the
 * device's primary context) invalidates the kept address, so this library
 * must not be called again in that process afterwards.
 * All calls share the one array: calls whose GPU work overlaps (on
 * different streams, or from different host threads) race on it and give
 * wrong results; serialise them. What a previous call left in the array does
 * not affect a call.
 */
ttt_status lact_swiglu_fwd_noalloc(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                                   const ttt_tensor* eta, const ttt_tensor* W1,
                                   const ttt_tensor* W2, const ttt_tensor* W3, int32_t chunk,
                                   int32_t update_rule, int32_t causal, const ttt_tensor* out,
                                   const ttt_tensor* W1_final, const ttt_tensor* W2_final,
                                   const ttt_tensor* W3_final, void* stream);

/*
 * Sliding-window causal softmax attention ("Test-Time Training Done Right"
 * review, section 3.1: window attention models the relations between tokens
 * within a fixed range; the pages give windows of 2K and 4K tokens):
 *   y_t = sum_{t-window < i <= t} softmax_i(q_t . k_i / sqrt(d)) v_i.
 *  q, k [B,H,T,d], v, out [B,H,T,d]: bf16, d in {64, 128, 256}
 *  window >= 1 (a window of T or more is plain causal attention)
 *  accumulate 0: out = y; 1: out = out + y (summed in fp32, rounded once)
 * mma.sync tensor-core tiles (bf16 operands, fp32 accumulation) with an
 * online softmax; fp32 tokens or other sizes -> TTT_ERR_UNSUPPORTED.
 */
ttt_status window_attention_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                                int32_t window, int32_t accumulate, const ttt_tensor* out,
                                void* stream);

/*
 * LaCT's hybrid block: the LaCT layer (causal, lact_swiglu_fwd) and window
 * attention on the same q, k, v, outputs summed (review, section 4: the
 * attention and the TTT layer share Q, K and V and their outputs are
 * combined; this library takes the sum). Arguments as lact_swiglu_fwd plus
 * `window`; bf16 with d in {64, 128, 256}.
 */
ttt_status lact_swiglu_window_fwd(const ttt_tensor* q, const ttt_tensor* k, const ttt_tensor* v,
                                  const ttt_tensor* eta, const ttt_tensor* W1,
                                  const ttt_tensor* W2, const ttt_tensor* W3, int32_t chunk,
                                  int32_t update_rule, int32_t window, const ttt_tensor* out,
                                  void* stream);

/* Static description of a status code (never NULL). */
const char* ttt_status_string(int32_t status);

/* Synchronises `stream`, returns the first device-side error recorded since
 * the last call (TTT_OK if none) and clears it. */
ttt_status ttt_get_device_status(void* stream);

/* Test hook of the failure handling: the next n stream-ordered scratch
 * allocations of the library (LaCT, the TTT-Linear backward, TTT-MLP) fail
 * as if the device were out of memory, so the calls return TTT_ERR_ALLOC
 * without launching anything. n = 0 turns it off. No GPU fault is involved. */
void ttt_test_fail_allocations(int32_t n);

/* Library version, as major*10000 + minor*100 + patch. */
int32_t ttt_version(void);

/*
 * Self-test of the failure detection: enqueues one CTA that waits on a
 * barrier nothing arrives at. The bounded wait gives up after its limit
 * (about 2 s), records TTT_ERR_TIMEOUT in the device status word and the
 * kernel returns, leaving the context usable; ttt_get_device_status() then
 * returns TTT_ERR_TIMEOUT (and clears it). Returns TTT_OK once launched.
 */
ttt_status ttt_selftest_wait_timeout(void* stream);

/*
 * Self-test of the debug-bounds build (the library compiled with
 * -DTTT_DEBUG_BOUNDS, libttt_b200_dbg.so): enqueues one CTA whose index check
 * fails by construction, without touching memory; ttt_get_device_status()
 * then returns TTT_ERR_BOUNDS (and clears it). In that build every kernel
 * index check that fails records TTT_ERR_BOUNDS the same way and skips the
 * access instead of trapping. Returns TTT_OK once launched, or
 * TTT_ERR_UNSUPPORTED from the normal build, whose checks are compiled out.
 */
ttt_status ttt_selftest_bounds(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TTT_B200_H */
