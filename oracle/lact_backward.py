"""fp64 CPU oracle for the LaCT layer's backward pass (training).

TEST INFRASTRUCTURE ONLY, like ``ttt_oracle``: nothing on the product path
may import, call or run it, and it shares no code with the CUDA path.

The LaCT forward of ``ttt_oracle.lact_swiglu`` is restated here step for step
in plain PyTorch fp64 CPU ops ([LaCT] "Test-Time Training Done Right" review:
section 3.2, SwiGLU fast weights and the eta-weighted negative inner-product
chunk loss; section 3.3, GD or Muon with Newton-Schulz, then L2 row
normalisation; section 4 / Figure 3, the apply/update order). The backward
pass is then the reverse-mode derivative of that restatement, taken by
autograd. It reaches through the fast-weight gradients themselves (second
order), the Newton-Schulz polynomial and the row renormalisation, whose
target norms are those of the initial weights.

Pins (``tests/test_oracle_backward.py``): this forward equals
``ttt_oracle.lact_swiglu``; the gradients match central finite differences
of ``ttt_oracle.lact_swiglu`` (numpy) along random directions; and with
eta = 0 they reduce to the closed-form SwiGLU gradients.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ttt_oracle as O


def _t(x, grad=False):
    return torch.tensor(np.asarray(x, dtype=np.float64), dtype=torch.float64, requires_grad=grad)


def _swiglu(W1, W2, W3, X):
    # f(x) = W2 (silu(W1 x) * W3 x) for each row x of X
    return (torch.nn.functional.silu(X @ W1.T) * (X @ W3.T)) @ W2.T


def _chunk_grads(W1, W2, W3, K, V, eta):
    # analytic gradients of sum_i eta_i * (-f(k_i) . v_i), as in the forward
    H1 = K @ W1.T
    H3 = K @ W3.T
    s = torch.sigmoid(H1)
    act = H1 * s * H3
    df = -eta[:, None] * V
    G2 = df.T @ act
    dact = df @ W2
    dH3 = dact * (H1 * s)
    dH1 = dact * H3 * (s * (1.0 + H1 * (1.0 - s)))
    return dH1.T @ K, G2, dH3.T @ K


def _ns5(G):
    a, b, c = O.NS_COEFFS
    X = G / (torch.linalg.norm(G) + O.NS_EPS)
    for _ in range(O.NS_STEPS):
        A = X @ X.T
        X = a * X + b * (A @ X) + c * (A @ (A @ X))
    return X


def _renorm(W, rho):
    n = torch.sqrt(torch.sum(W * W, dim=-1))
    safe = torch.where(n > 0, n, torch.ones_like(n))
    scale = torch.where(n > 0, rho / safe, torch.ones_like(n))
    return W * scale[:, None]


def lact_swiglu_torch(q, k, v, eta, W1, W2, W3, chunk, update_rule, causal):
    """The LaCT forward for one (batch, head): q, k [T,dk], v [T,dv], eta [T],
    W1, W3 [dh,dk], W2 [dv,dh], all torch fp64. Returns (y, W1, W2, W3)."""
    T = q.shape[0]
    rho = [torch.sqrt(torch.sum(W * W, dim=-1)) for W in (W1, W2, W3)]
    w1, w2, w3 = W1, W2, W3
    ys = []
    for s in range(0, T, chunk):
        e = min(s + chunk, T)
        if causal:
            ys.append(_swiglu(w1, w2, w3, q[s:e]))
        g1, g2, g3 = _chunk_grads(w1, w2, w3, k[s:e], v[s:e], eta[s:e])
        if update_rule == O.UPDATE_MUON:
            g1, g2, g3 = _ns5(g1), _ns5(g2), _ns5(g3)
        elif update_rule != O.UPDATE_GD:
            raise ValueError(update_rule)
        w1 = _renorm(w1 - g1, rho[0])
        w2 = _renorm(w2 - g2, rho[1])
        w3 = _renorm(w3 - g3, rho[2])
        if not causal:
            ys.append(_swiglu(w1, w2, w3, q[s:e]))
    y = torch.cat(ys) if ys else torch.zeros((0, v.shape[1]), dtype=torch.float64)
    return y, w1, w2, w3


def lact_swiglu_bwd(q, k, v, eta, W1, W2, W3, chunk, update_rule, causal, dy, dW_final=None):
    """Gradients of a scalar objective through the LaCT layer, given
    dL/dy [B,H,T,dv] and optionally dL/d(final weights) as a tuple
    (dW1 [B,H,dh,dk], dW2 [B,H,dv,dh], dW3 [B,H,dh,dk]).

    Returns (dq, dk, dv, deta, dW1, dW2, dW3). The weight gradients have the
    shape of the given weights: summed over the batch when the weights are
    shared by it ([H,...])."""
    q, k, v, eta, dy = (np.asarray(x, dtype=np.float64) for x in (q, k, v, eta, dy))
    B, H, T, _ = q.shape
    Ws = [np.asarray(W, dtype=np.float64) for W in (W1, W2, W3)]
    shared = Ws[0].ndim == 3
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(eta)]
    dWs = [np.zeros_like(W) for W in Ws]
    for bi in range(B):
        for h in range(H):
            tq, tk, tv, te = (_t(x[bi, h], True) for x in (q, k, v, eta))
            tw = [_t(W[h] if shared else W[bi, h], True) for W in Ws]
            y, f1, f2, f3 = lact_swiglu_torch(tq, tk, tv, te, *tw, chunk, update_rule, causal)
            obj = torch.sum(y * _t(dy[bi, h]))
            if dW_final is not None:
                for f, d in zip((f1, f2, f3), dW_final):
                    obj = obj + torch.sum(f * _t(np.asarray(d)[bi, h]))
            grads = torch.autograd.grad(obj, [tq, tk, tv, te] + tw, allow_unused=True)
            for n in range(4):
                if grads[n] is not None:
                    out[n][bi, h] = grads[n].numpy()
            for n in range(3):
                g = grads[4 + n]
                if g is None:
                    continue
                if shared:
                    dWs[n][h] += g.numpy()
                else:
                    dWs[n][bi, h] = g.numpy()
    return (*out, *dWs)
