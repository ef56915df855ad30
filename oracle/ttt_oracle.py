"""Plain fp64 CPU oracle for the chunked TTT-layer forward pass.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference leg use it. It shares no code with the CUDA path
(``linear_attention_ttt_b200/csrc``); the two only receive the same seeded
inputs from ``linear_attention_ttt_b200.synth``.

Everything here is written from the pages' definitions, in float64, with numpy
matmul/einsum as the only library primitive, and with no blocking, fusion or
reordering beyond what each definition states. Sources (page title, section):

* [TTT] "Test-Time Training (TTT)" summary (eommydocs): sections
  "Linear Attention", "TTT 정의" (definition), "예시 1: Linear Attention 유도"
  (inner-product loss), "예시 2: DeltaNet 유도" (MSE loss), "TTT-Linear",
  "병렬화: Mini-batch Gradient Descent", "Arithmetic Intensity 분석".
* [LaCT] "Test-Time Training Done Right" review (iplexlaw blog): section 3.2
  (SwiGLU fast weights, negative inner-product loss, per-token learning rates,
  summed chunk gradient), section 3.3 (GD / Muon with Newton-Schulz, L2
  normalisation after the update), section 4 and Figure 3 (apply/update order).
* [KVB] "Test-Time Training with KV Binding Is Secretly Linear Attention"
  (abstract): TTT with KV binding as a learned linear-attention operator.

Readings taken where the pages are silent or disagree (each is also listed in
the design notes):
* MSE scale is 1/2||kW - v||^2 (the DeltaNet derivation), so the per-token
  gradient is k^T (kW - v).
* The query of token t sees the update of token t: W_t includes i = t
  (the definition y_t = f(q_t, W_t) and the inclusive sum i = t'..t of the
  mini-batch rule).
* TTT-Linear uses row vectors, f(x) = xW with W of shape (d_in, d_out).
  LaCT uses column vectors, f(x) = W2 (silu(W1 x) * W3 x), weights stored
  (out, in).
* LaCT: eta_i weights token i's loss; the update is W <- W - G with G the
  eta-weighted sum (GD), or W <- W - NS5(G) (Muon, unit step). Newton-Schulz
  starts from G / (||G||_F + 1e-7). After each update every row of W1, W3
  (a hidden unit, over d_in) and of W2 (an output unit, over hidden) is
  rescaled to the L2 norm that row had in the initial weights of the call;
  a zero row is left as is.
* LaCT causal order: apply W_{c-1} to chunk c's queries, then update with
  chunk c. Non-causal: update with chunk c, then apply to chunk c.

Layouts: q, k [B,H,T,dk]; v [B,H,T,dv]; eta [B,H,T]; TTT-Linear W0 [H,dk,dv]
(shared over the batch) or [B,H,dk,dv]; LaCT W1, W3 [H,dh,dk], W2 [H,dv,dh]
(or with a leading B). Outputs y [B,H,T,dv].

Parity status: every function below is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (the forward pass) and
``tests/test_oracle_backward.py`` (the TTT-Linear backward pass) except where
its docstring says otherwise.
"""
from __future__ import annotations

import numpy as np

LOSS_MSE = 0
LOSS_NEG_DOT = 1
UPDATE_GD = 0
UPDATE_MUON = 1
UPDATE_MOMENTUM = 2

# Newton-Schulz quintic coefficients (a, b, c) and the normalisation epsilon.
NS_COEFFS = (3.4445, -4.7750, 2.0315)
NS_STEPS = 5
NS_EPS = 1e-7


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _broadcast_state(W, B):
    """Per-head initial state [H,...] is shared by every sequence in the batch
    ([TTT] Python example: the per-head init is expanded over the batch)."""
    W = _f64(W)
    return np.broadcast_to(W, (B,) + W.shape).copy() if W.ndim == 3 else W.copy()


# ----------------------------------------------------------------------------
# Per-token losses and gradients of TTT-Linear, f(k; W) = k W.
# ----------------------------------------------------------------------------

def loss_value(W, k, v, loss):
    """Scalar loss of one token for one head. W [dk,dv], k [dk], v [dv].

    MSE ([TTT] "예시 2"): 1/2 ||kW - v||^2.
    Inner product ([TTT] "예시 1"): -(kW) . v.
    """
    W, k, v = _f64(W), _f64(k), _f64(v)
    pred = k @ W
    if loss == LOSS_MSE:
        return 0.5 * float(np.sum((pred - v) ** 2))
    if loss == LOSS_NEG_DOT:
        return -float(pred @ v)
    raise ValueError(loss)


def loss_grad(W, k, v, loss):
    """dL/dW for one token, batched over leading dims.

    W [...,dk,dv], k [...,dk], v [...,dv] -> [...,dk,dv].
    MSE: k^T (kW - v)  ([TTT] "예시 2").  Inner product: -k^T v ([TTT] "예시 1").
    """
    W, k, v = _f64(W), _f64(k), _f64(v)
    if loss == LOSS_MSE:
        err = np.einsum("...a,...ab->...b", k, W) - v
        return np.einsum("...a,...b->...ab", k, err)
    if loss == LOSS_NEG_DOT:
        return -np.einsum("...a,...b->...ab", k, v)
    raise ValueError(loss)


# ----------------------------------------------------------------------------
# TTT-Linear: token recurrence, mini-batch GD (the definition), dual form.
# ----------------------------------------------------------------------------

def ttt_linear_token_recurrence(q, k, v, eta, W0, loss):
    """One gradient step per token ([TTT] "TTT 정의"):
    W_t = W_{t-1} - eta_t dL(W_{t-1}; k_t, v_t)/dW,  y_t = q_t W_t.
    Returns (y [B,H,T,dv], W_T [B,H,dk,dv])."""
    q, k, v, eta = _f64(q), _f64(k), _f64(v), _f64(eta)
    B, H, T, _ = q.shape
    W = _broadcast_state(W0, B)
    y = np.zeros((B, H, T, v.shape[-1]))
    for t in range(T):
        W = W - eta[:, :, t, None, None] * loss_grad(W, k[:, :, t], v[:, :, t], loss)
        y[:, :, t] = np.einsum("zha,zhac->zhc", q[:, :, t], W)
    return y, W


def ttt_linear_minibatch(q, k, v, eta, W0, chunk, loss):
    """Mini-batch gradient descent, the definition ([TTT] "병렬화: Mini-batch
    Gradient Descent"): with t' = t - (t mod b) the chunk start,
        W_t = W_{t'} - sum_{i=t'}^{t} eta_i dL(W_{t'}; k_i, v_i)/dW,
        y_t = q_t W_t.
    Every gradient of a chunk is taken at the chunk-start weights W_{t'}; the
    next chunk starts from the weights of the chunk's last token. A last,
    shorter chunk follows the same rule. Returns (y, W_final)."""
    q, k, v, eta = _f64(q), _f64(k), _f64(v), _f64(eta)
    B, H, T, _ = q.shape
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    W = _broadcast_state(W0, B)
    y = np.zeros((B, H, T, v.shape[-1]))
    for s in range(0, T, chunk):
        W_start = W.copy()
        acc = np.zeros_like(W_start)
        for t in range(s, min(s + chunk, T)):
            acc += eta[:, :, t, None, None] * loss_grad(W_start, k[:, :, t], v[:, :, t], loss)
            W = W_start - acc
            y[:, :, t] = np.einsum("zha,zhac->zhc", q[:, :, t], W)
    return y, W


def ttt_linear_dual(q, k, v, eta, W0, chunk, loss):
    """The dual (parallel) form of one mini-batch chunk, per head, with
    Q, K [b,dk], V [b,dv], N = diag(eta) and tril keeping i <= t:
      MSE:            E = K W - V,   Y = Q W - (tril(Q K^T) N) E,
                      W <- W - K^T N E
      inner product:  Y = Q W + (tril(Q K^T) N) V,   W <- W + K^T N V
    (the closed form of the mini-batch rule stated in [KVB]'s "fully parallel
    formulation" sense; it equals ``ttt_linear_minibatch`` exactly, which the
    pins check). Returns (y, W_final)."""
    q, k, v, eta = _f64(q), _f64(k), _f64(v), _f64(eta)
    B, H, T, _ = q.shape
    W = _broadcast_state(W0, B)
    y = np.zeros((B, H, T, v.shape[-1]))
    for s in range(0, T, chunk):
        e = min(s + chunk, T)
        Q, K, V, n = q[:, :, s:e], k[:, :, s:e], v[:, :, s:e], eta[:, :, s:e]
        A = np.tril(Q @ np.swapaxes(K, -1, -2)) * n[:, :, None, :]
        if loss == LOSS_MSE:
            E = K @ W - V
            y[:, :, s:e] = Q @ W - A @ E
            W = W - np.swapaxes(K, -1, -2) @ (n[..., None] * E)
        elif loss == LOSS_NEG_DOT:
            y[:, :, s:e] = Q @ W + A @ V
            W = W + np.swapaxes(K, -1, -2) @ (n[..., None] * V)
        else:
            raise ValueError(loss)
    return y, W


def linear_attention(q, k, v, eta, S0):
    """Linear attention recurrence ([TTT] "Linear Attention", with the
    per-token weight of "예시 1"): S_t = S_{t-1} + eta_t k_t^T v_t,
    y_t = q_t S_t. Returns (y, S_T)."""
    q, k, v, eta = _f64(q), _f64(k), _f64(v), _f64(eta)
    B, H, T, _ = q.shape
    S = _broadcast_state(S0, B)
    y = np.zeros((B, H, T, v.shape[-1]))
    for t in range(T):
        S = S + eta[:, :, t, None, None] * np.einsum("zha,zhc->zhac", k[:, :, t], v[:, :, t])
        y[:, :, t] = np.einsum("zha,zhac->zhc", q[:, :, t], S)
    return y, S


# ----------------------------------------------------------------------------
# TTT-Linear backward: the reverse chunk scan (training).
# ----------------------------------------------------------------------------

def ttt_linear_minibatch_bwd(q, k, v, eta, W0, chunk, loss, dy, dW_final=None):
    """Gradients of a scalar objective through ``ttt_linear_minibatch``, given
    dL/dy [B,H,T,dv] and dL/dW_final [B,H,dk,dv] (None means zero).

    The chain rule written out for the mini-batch rule ([TTT] "병렬화:
    Mini-batch Gradient Descent"). In a chunk with start weights W, token t
    uses W_t = W - sum_{i<=t} eta_i g_i(W) and y_t = q_t W_t, and the chunk's
    last W_t starts the next chunk. With U_t = dL/dW_t = q_t^T dy_t (plus, at
    the chunk's last token, the gradient of the next chunk's start) and
    R_i = sum of U_t over t >= i in the chunk:
      dq_t    = dy_t W_t^T
      deta_i  = -<R_i, g_i(W)>
      and Gamma_i = -eta_i R_i flows into g_i:
        MSE, g_i = k_i^T e_i with e_i = k_i W - v_i:
          de_i = k_i Gamma_i,  dk_i = e_i Gamma_i^T + de_i W^T,
          dv_i = -de_i,        dL/dW gains k_i^T de_i;
        inner product, g_i = -k_i^T v_i:
          dk_i = -v_i Gamma_i^T,  dv_i = -k_i Gamma_i.
      dL/dW (the chunk start) = sum_t U_t (+ the MSE terms), carried back to
      the previous chunk.
    Returns (dq, dk, dv, deta, dW0); dW0 is summed over the batch when W0 is
    shared by it ([H,dk,dv])."""
    q, k, v, eta, dy = map(_f64, (q, k, v, eta, dy))
    B, H, T, _ = q.shape
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    if loss not in (LOSS_MSE, LOSS_NEG_DOT):
        raise ValueError(loss)
    # forward: the start weights of every chunk
    W = _broadcast_state(W0, B)
    starts = list(range(0, T, chunk))
    W_start = []
    for s in starts:
        W_start.append(W.copy())
        for i in range(s, min(s + chunk, T)):
            W = W - eta[:, :, i, None, None] * loss_grad(W_start[-1], k[:, :, i], v[:, :, i], loss)
    G = np.zeros_like(W) if dW_final is None else _f64(dW_final).copy()
    dq, dk, dv, deta = (np.zeros_like(x) for x in (q, k, v, eta))
    for ci in reversed(range(len(starts))):
        s, Ws = starts[ci], W_start[ci]
        e = min(s + chunk, T)
        g, Wt, acc = [], [], np.zeros_like(Ws)
        for i in range(s, e):
            g.append(loss_grad(Ws, k[:, :, i], v[:, :, i], loss))
            acc = acc + eta[:, :, i, None, None] * g[-1]
            Wt.append(Ws - acc)
        R = np.zeros_like(Ws)
        dWs = np.zeros_like(Ws)
        for idx in reversed(range(e - s)):
            t = s + idx
            U = np.einsum("zha,zhc->zhac", q[:, :, t], dy[:, :, t])
            if t == e - 1:
                U = U + G
            dq[:, :, t] = np.einsum("zhc,zhac->zha", dy[:, :, t], Wt[idx])
            R = R + U
            dWs = dWs + U
            deta[:, :, t] = -np.einsum("zhac,zhac->zh", R, g[idx])
            Gam = -eta[:, :, t, None, None] * R
            if loss == LOSS_MSE:
                err = np.einsum("zha,zhac->zhc", k[:, :, t], Ws) - v[:, :, t]
                de = np.einsum("zha,zhac->zhc", k[:, :, t], Gam)
                dk[:, :, t] = (np.einsum("zhac,zhc->zha", Gam, err) +
                               np.einsum("zhc,zhac->zha", de, Ws))
                dv[:, :, t] = -de
                dWs = dWs + np.einsum("zha,zhc->zhac", k[:, :, t], de)
            else:
                dk[:, :, t] = -np.einsum("zhac,zhc->zha", Gam, v[:, :, t])
                dv[:, :, t] = -np.einsum("zha,zhac->zhc", k[:, :, t], Gam)
        G = dWs
    dW0 = G.sum(axis=0) if _f64(W0).ndim == 3 else G
    return dq, dk, dv, deta, dW0


# ----------------------------------------------------------------------------
# TTT-MLP (the scope table's "next" row f3): a two-layer ReLU MLP fast weight.
# ----------------------------------------------------------------------------

def mlp_apply(W1, b1, W2, b2, x):
    """f(x) = W2 ReLU(W1 x + b1) + b2 ([TTT] "TTT-MLP"), for the rows x of X
    [n, dk]; W1 [dh, dk], b1 [dh], W2 [dv, dh], b2 [dv]. Returns [n, dv]."""
    x = _f64(x)
    return np.maximum(x @ _f64(W1).T + _f64(b1), 0.0) @ _f64(W2).T + _f64(b2)


def mlp_loss(W1, b1, W2, b2, k, v):
    """Per-token loss 1/2 ||f(k) - v||^2 (the MSE reading of TTT-Linear,
    applied to the MLP fast weight)."""
    r = mlp_apply(W1, b1, W2, b2, _f64(k)[None])[0] - _f64(v)
    return 0.5 * float(r @ r)


def mlp_grads(W1, b1, W2, b2, k, v):
    """Gradients of ``mlp_loss`` for one token: with h = W1 k + b1,
    a = ReLU(h), r = W2 a + b2 - v: db2 = r, dW2 = r a^T, dh = (W2^T r) [h > 0]
    (derivative 0 at h = 0), db1 = dh, dW1 = dh k^T."""
    W1, b1, W2, b2, k, v = map(_f64, (W1, b1, W2, b2, k, v))
    h = W1 @ k + b1
    a = np.maximum(h, 0.0)
    r = W2 @ a + b2 - v
    dh = (W2.T @ r) * (h > 0)
    return np.outer(dh, k), dh, np.outer(r, a), r


def ttt_mlp_token_recurrence(q, k, v, eta, W1, b1, W2, b2):
    """One gradient step per token ([TTT] "TTT 정의" with the MLP of
    "TTT-MLP"): W_t = W_{t-1} - eta_t grad(W_{t-1}; k_t, v_t), y_t = f(q_t; W_t),
    for all four parameters. Single sequence: q, k [T, dk], v [T, dv], eta [T].
    Returns (y [T, dv], (W1, b1, W2, b2) after the last token)."""
    P = [_f64(x).copy() for x in (W1, b1, W2, b2)]
    q, k, v, eta = map(_f64, (q, k, v, eta))
    y = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        g = mlp_grads(*P, k[t], v[t])
        P = [p - eta[t] * gi for p, gi in zip(P, g)]
        y[t] = mlp_apply(*P, q[t][None])[0]
    return y, tuple(P)


def ttt_mlp_minibatch(q, k, v, eta, W1, b1, W2, b2, chunk):
    """Mini-batch gradient descent on the MLP fast weight, the rule of
    [TTT] "병렬화: Mini-batch Gradient Descent" for every parameter: with t'
    the chunk start, P_t = P_{t'} - sum_{i=t'}^{t} eta_i grad(P_{t'}; k_i, v_i)
    and y_t = f(q_t; P_t). Single sequence, as ``ttt_mlp_token_recurrence``.
    The pages print no numbers for TTT-MLP; the pins are the closed forms,
    invariants and derivative checks of ``tests/test_oracle_ttt_mlp.py``."""
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    P = [_f64(x).copy() for x in (W1, b1, W2, b2)]
    q, k, v, eta = map(_f64, (q, k, v, eta))
    T = q.shape[0]
    y = np.zeros((T, v.shape[1]))
    for s in range(0, T, chunk):
        start = [p.copy() for p in P]
        acc = [np.zeros_like(p) for p in P]
        for t in range(s, min(s + chunk, T)):
            g = mlp_grads(*start, k[t], v[t])
            acc = [a + eta[t] * gi for a, gi in zip(acc, g)]
            P = [p0 - a for p0, a in zip(start, acc)]
            y[t] = mlp_apply(*P, q[t][None])[0]
    return y, tuple(P)


# ----------------------------------------------------------------------------
# Sliding-window attention beside LaCT (the scope table's "next" row f4).
# ----------------------------------------------------------------------------

def sliding_window_attention(q, k, v, window):
    """Causal softmax attention over the last `window` tokens ([LaCT] 3.1:
    window attention computes the relations between tokens within a fixed
    range): y_t = sum_{t-window < i <= t} softmax_i(q_t . k_i / sqrt(d)) v_i.
    Single sequence: q, k [T, d], v [T, dv]. Returns [T, dv]."""
    q, k, v = map(_f64, (q, k, v))
    if window < 1:
        raise ValueError("window must be >= 1")
    T, d = q.shape
    y = np.zeros((T, v.shape[1]))
    for t in range(T):
        lo = max(0, t - window + 1)
        s = k[lo:t + 1] @ q[t] / np.sqrt(d)
        p = np.exp(s - s.max())
        y[t] = (p / p.sum()) @ v[lo:t + 1]
    return y


def lact_with_window_attention(q, k, v, eta, W1, W2, W3, chunk, update_rule, window):
    """The LaCT layer with window attention beside it, both on the same q, k,
    v ([LaCT] 4: attention and TTT share Q, K, V and their outputs are
    combined), combined by summing the two outputs (causal order).
    Single sequence, weights [dh, d] / [d, dh]. Returns [T, dv]."""
    y, *_ = lact_swiglu(_f64(q)[None, None], _f64(k)[None, None], _f64(v)[None, None],
                        _f64(eta)[None, None], _f64(W1)[None], _f64(W2)[None], _f64(W3)[None],
                        chunk, update_rule, 1)
    return y[0, 0] + sliding_window_attention(q, k, v, window)


def arithmetic_intensity(b, h):
    """[TTT] "Arithmetic Intensity 분석": fast weight h x h, chunk input b x h,
    r = 2 h^2 b / (2 h^2 + 4 h b)  (= b / (1 + 2b/h), bounded by min(h/2, b))."""
    return 2.0 * h * h * b / (2.0 * h * h + 4.0 * h * b)


# ----------------------------------------------------------------------------
# LaCT: SwiGLU fast-weight MLP, chunked GD / Muon, L2 row renormalisation.
# ----------------------------------------------------------------------------

def sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * _f64(x)))


def silu(x):
    x = _f64(x)
    return x * sigmoid(x)


def silu_grad(x):
    s = sigmoid(x)
    return s * (1.0 + _f64(x) * (1.0 - s))


def swiglu(W1, W2, W3, X):
    """f(x) = W2 (silu(W1 x) * W3 x) for each row x of X [n,dk] ([LaCT] 3.2:
    three-matrix SwiGLU MLP). W1, W3 [dh,dk]; W2 [dv,dh]. Returns [n,dv]."""
    W1, W2, W3, X = _f64(W1), _f64(W2), _f64(W3), _f64(X)
    return (silu(X @ W1.T) * (X @ W3.T)) @ W2.T


def lact_loss(W1, W2, W3, K, V, eta):
    """Chunk loss sum_i eta_i * (-f(k_i) . v_i) ([LaCT] 3.2: negative inner
    product, each token weighted by its learning rate, summed over the chunk)."""
    return -float(np.sum(_f64(eta)[:, None] * swiglu(W1, W2, W3, K) * _f64(V)))


def lact_grads(W1, W2, W3, K, V, eta):
    """Gradients of ``lact_loss`` with respect to W1, W2, W3 (chain rule).
    K [n,dk], V [n,dv], eta [n]. Returns (G1 [dh,dk], G2 [dv,dh], G3 [dh,dk])."""
    W1, W2, W3, K, V, eta = map(_f64, (W1, W2, W3, K, V, eta))
    H1 = K @ W1.T
    H3 = K @ W3.T
    act = silu(H1) * H3
    df = -eta[:, None] * V                 # dL/df_i
    G2 = df.T @ act                        # dL/dW2
    dact = df @ W2                         # dL/d act_i
    dH3 = dact * silu(H1)
    dH1 = dact * H3 * silu_grad(H1)
    G1 = dH1.T @ K
    G3 = dH3.T @ K
    return G1, G2, G3


def newton_schulz5(G, coeffs=NS_COEFFS, steps=NS_STEPS, eps=NS_EPS):
    """Muon's orthogonalisation ([LaCT] 3.3: the matrix gradient is
    transformed by Newton-Schulz iteration): X0 = G / (||G||_F + eps), then
    `steps` times X <- a X + b (X X^T) X + c (X X^T)^2 X."""
    a, b, c = coeffs
    X = _f64(G) / (np.linalg.norm(_f64(G)) + eps)
    for _ in range(steps):
        A = X @ X.T
        X = a * X + b * (A @ X) + c * (A @ (A @ X))
    return X


def row_norms(W):
    return np.sqrt(np.sum(_f64(W) ** 2, axis=-1))


def renorm_rows(W, rho):
    """Rescale each row of W to the target L2 norm rho ([LaCT] 3.3: L2
    normalisation of the fast weights after the update). Zero rows stay zero."""
    W = _f64(W)
    n = row_norms(W)
    scale = np.where(n > 0, _f64(rho) / np.where(n > 0, n, 1.0), 1.0)
    return W * scale[..., None]


def lact_swiglu(q, k, v, eta, W1, W2, W3, chunk, update_rule=UPDATE_GD, causal=1):
    """LaCT layer forward ([LaCT] 3.2-3.3, 4 / Figure 3), per (batch, head):
    for each chunk c of `chunk` tokens (the last may be shorter)
      causal=1: Y_c = f_{W}(Q_c) with the weights before chunk c, then update;
      causal=0: update with chunk c first, then Y_c = f_{W}(Q_c).
    Update: G = grads of sum_i eta_i (-f(k_i) . v_i) at the current weights;
    Muon replaces each of G1, G2, G3 by NS5 of it; W <- W - G; then rows are
    renormalised to the initial row norms.
    Returns (y [B,H,T,dv], W1_final, W2_final, W3_final) with finals [B,H,...]."""
    q, k, v, eta = map(_f64, (q, k, v, eta))
    B, H, T, _ = q.shape
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    Ws = [_broadcast_state(W, B) for W in (W1, W2, W3)]
    y = np.zeros((B, H, T, v.shape[-1]))
    for bi in range(B):
        for h in range(H):
            w1, w2, w3 = (W[bi, h].copy() for W in Ws)
            rho = [row_norms(w) for w in (w1, w2, w3)]
            for s in range(0, T, chunk):
                e = min(s + chunk, T)
                if causal:
                    y[bi, h, s:e] = swiglu(w1, w2, w3, q[bi, h, s:e])
                g1, g2, g3 = lact_grads(w1, w2, w3, k[bi, h, s:e], v[bi, h, s:e], eta[bi, h, s:e])
                if update_rule == UPDATE_MUON:
                    g1, g2, g3 = newton_schulz5(g1), newton_schulz5(g2), newton_schulz5(g3)
                elif update_rule != UPDATE_GD:
                    raise ValueError(update_rule)
                w1 = renorm_rows(w1 - g1, rho[0])
                w2 = renorm_rows(w2 - g2, rho[1])
                w3 = renorm_rows(w3 - g3, rho[2])
                if not causal:
                    y[bi, h, s:e] = swiglu(w1, w2, w3, q[bi, h, s:e])
            Ws[0][bi, h], Ws[1][bi, h], Ws[2][bi, h] = w1, w2, w3
    return y, Ws[0], Ws[1], Ws[2]


def lact_swiglu_momentum(q, k, v, eta, W1, W2, W3, chunk, beta, causal=1, M0=None):
    """LaCT with the momentum update ([LaCT] 3.3 names GD, momentum and Muon
    as the compared update rules, and prints no formula for momentum). The
    reading taken is heavy-ball momentum over chunk gradients, per matrix:
      M <- beta * M + G,   W <- renorm(W - M),   M = 0 before the first chunk
    (or M0), with G the eta-weighted summed gradient of ``lact_swiglu`` and
    the same apply/update order and row renormalisation. beta = 0 is GD.
    Returns (y, W1_final, W2_final, W3_final, (M1, M2, M3)), all [B,H,...]."""
    q, k, v, eta = map(_f64, (q, k, v, eta))
    B, H, T, _ = q.shape
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    Ws = [_broadcast_state(W, B) for W in (W1, W2, W3)]
    Ms = [np.zeros_like(W) for W in Ws] if M0 is None else [_broadcast_state(M, B) for M in M0]
    y = np.zeros((B, H, T, v.shape[-1]))
    for bi in range(B):
        for h in range(H):
            w = [W[bi, h].copy() for W in Ws]
            m = [M[bi, h].copy() for M in Ms]
            rho = [row_norms(x) for x in w]
            for s in range(0, T, chunk):
                e = min(s + chunk, T)
                if causal:
                    y[bi, h, s:e] = swiglu(*w, q[bi, h, s:e])
                g = lact_grads(*w, k[bi, h, s:e], v[bi, h, s:e], eta[bi, h, s:e])
                for i in range(3):
                    m[i] = beta * m[i] + g[i]
                    w[i] = renorm_rows(w[i] - m[i], rho[i])
                if not causal:
                    y[bi, h, s:e] = swiglu(*w, q[bi, h, s:e])
            for i in range(3):
                Ws[i][bi, h] = w[i]
                Ms[i][bi, h] = m[i]
    return y, Ws[0], Ws[1], Ws[2], tuple(Ms)


def lact_swiglu_prefix(q, k, v, eta, W1, W2, W3, chunk, update_rule, n_chunks, bh):
    """Outputs of the first `n_chunks` chunks of one (batch, head) pair `bh`,
    computed by running ``lact_swiglu`` on the truncated sequence. Causal
    outputs of chunk c depend only on chunks <= c, so this is exact; it lets
    full-size runs be checked on a prefix."""
    bi, h = bh
    T = min(q.shape[2], n_chunks * chunk)
    sl = (slice(bi, bi + 1), slice(h, h + 1), slice(0, T))
    pick = (lambda W: W[h:h + 1]) if np.ndim(W1) == 3 else (lambda W: W[bi:bi + 1, h:h + 1])
    y, *_ = lact_swiglu(q[sl], k[sl], v[sl], eta[sl], pick(W1), pick(W2), pick(W3),
                        chunk, update_rule, 1)
    return y[0, 0]
