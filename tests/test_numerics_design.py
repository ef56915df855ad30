"""Rounding design of the inner-product kernel, checked with a numpy model of
where its tensor-core products round to bf16 (CPU).

The kernel computes, per 64-token tile, P = bf16(tril(Q K^T)) and
Vt = bf16(diag(eta) V), and Y = Q bf16(S) + P Vt with fp32 accumulation. A
variant that folds eta into K before the score (P = bf16(tril(Q bf16(eta K)^T)))
rounds every k element first, so a row whose q.k nearly cancels loses its
relative accuracy. On the linear-attention workload's data the first token
of (batch 2, head 10) is such a row. This test keeps that lesson: the
eta-on-V rounding stays inside the bf16 tolerance there, the eta-on-K one
does not.
"""
import numpy as np

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import synth
from tests.gpu_util import TOL_BF16_ROW


def bf16(x):
    return synth.round_to_bf16(np.asarray(x, np.float32)).astype(np.float32)


def model(q, k, v, eta, eta_on_v, TT=64):
    T = q.shape[0]
    S = np.zeros((q.shape[1], v.shape[1]), np.float32)
    y = np.zeros((T, v.shape[1]), np.float32)
    for a in range(0, T, TT):
        Q, K, V, e = q[a:a + TT], k[a:a + TT], v[a:a + TT], eta[a:a + TT]
        if eta_on_v:
            P = bf16(np.tril(Q @ K.T))
            Vt = bf16(e[:, None] * V)
            Kt = K
        else:
            Kt = bf16(e[:, None] * K)
            P = bf16(np.tril(Q @ Kt.T))
            Vt = V
        y[a:a + TT] = bf16(Q @ bf16(S) + P @ Vt)
        S = S + Kt.T @ Vt
    return y


def worst_row(y, o):
    return float(np.max(np.abs(y - o).max(-1) / np.abs(o).max(-1)))


def test_eta_scales_v_not_k():
    w = synth.config(2)
    bh = (2, 10)
    T = 512  # the rows in question are at the start of the sequence
    f = lambda x: np.asarray(x[bh[0], bh[1], :T], np.float32)
    q, k, v, eta = f(w.q), f(w.k), f(w.v), f(w.eta)
    yo, _ = O.linear_attention(q[None, None], k[None, None], v[None, None], eta[None, None],
                               np.zeros((1, 128, 128)))
    o = yo[0, 0]
    good = worst_row(model(q, k, v, eta, eta_on_v=True), o)
    bad = worst_row(model(q, k, v, eta, eta_on_v=False), o)
    assert good <= TOL_BF16_ROW, good
    assert bad > TOL_BF16_ROW, bad
