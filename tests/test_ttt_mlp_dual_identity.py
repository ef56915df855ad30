"""Dual (chunk-parallel) form of TTT-MLP equals the oracle's mini-batch rule
(fp64, CPU). It is the form a kernel would use, and a check of the oracle by
a different algorithm.

Within a chunk with start parameters (W1, b1, W2, b2), every gradient is taken
at the start parameters, so for key token i: h_i = W1 k_i + b1,
a_i = ReLU(h_i), r_i = W2 a_i + b2 - v_i, g_i = (W2^T r_i) [h_i > 0]. Token
t's parameters are the start ones minus the eta-weighted sums over i <= t of
(g_i k_i^T, g_i, r_i a_i^T, r_i), so with N = diag(eta), L = tril(ones) N and
the rows of G, R, A, K as the g_i, r_i, a_i, k_i:
    Z  = Q W1^T + b1 - (tril(Q K^T) N) G - L G       (hidden pre-activations)
    Y  = ReLU(Z) W2^T + b2 - (tril(ReLU(Z) A^T) N) R - L R
and the chunk's end parameters are the start ones minus the full sums.
"""
import numpy as np
import pytest

from oracle import ttt_oracle as O


def dual_form(q, k, v, eta, W1, b1, W2, b2, chunk):
    T = q.shape[0]
    y = np.zeros((T, v.shape[1]))
    for s in range(0, T, chunk):
        e = min(s + chunk, T)
        Q, K, V, n = q[s:e], k[s:e], v[s:e], eta[s:e]
        H = K @ W1.T + b1
        A = np.maximum(H, 0.0)
        R = A @ W2.T + b2 - V
        G = (R @ W2) * (H > 0)
        L = np.tril(np.ones((e - s, e - s))) * n[None, :]
        Z = Q @ W1.T + b1 - (np.tril(Q @ K.T) * n[None, :]) @ G - L @ G
        Aq = np.maximum(Z, 0.0)
        y[s:e] = Aq @ W2.T + b2 - (np.tril(Aq @ A.T) * n[None, :]) @ R - L @ R
        W1 = W1 - (n[:, None] * G).T @ K
        b1 = b1 - n @ G
        W2 = W2 - (n[:, None] * R).T @ A
        b2 = b2 - n @ R
    return y, (W1, b1, W2, b2)


@pytest.mark.parametrize("chunk,T", [(1, 7), (3, 10), (8, 8), (5, 23), (32, 20)])
def test_dual_form_equals_the_minibatch_rule(chunk, T):
    rng = np.random.default_rng(chunk * 7 + T)
    dk, dh, dv = 4, 6, 3
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    eta = 0.1 * (0.5 + rng.random(T))
    P = (rng.standard_normal((dh, dk)) / 2, 0.1 * rng.standard_normal(dh),
         rng.standard_normal((dv, dh)) / 2, 0.1 * rng.standard_normal(dv))
    y, F = dual_form(q, k, v, eta, *P, chunk)
    yo, Fo = O.ttt_mlp_minibatch(q, k, v, eta, *P, chunk)
    np.testing.assert_allclose(y, yo, rtol=1e-11, atol=1e-12)
    for a, b in zip(F, Fo):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)
