"""Pins of the LaCT momentum oracle (the scope table's "next" row f2), CPU only.

The pages list momentum beside GD and Muon as LaCT update rules without a
formula. The reading pinned here: heavy-ball momentum on the chunk gradients,
M <- beta M + G, W <- renorm(W - M), M starting at zero.
"""
import numpy as np
import pytest

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import synth


def case(T=20, chunk=5, seed=3, B=1, H=2, d=4, dh=6):
    return synth.make_lact(B, H, T, d, dh, chunk, O.UPDATE_GD, seed, dtype=synth.F32,
                           eta_scale=0.05)


@pytest.mark.parametrize("causal", [1, 0])
def test_zero_beta_is_gd(causal):
    w = case()
    args = (w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, w.chunk)
    y, F1, F2, F3, _ = O.lact_swiglu_momentum(*args, 0.0, causal)
    yg, G1, G2, G3 = O.lact_swiglu(*args, O.UPDATE_GD, causal)
    np.testing.assert_array_equal(y, yg)
    for a, b in zip((F1, F2, F3), (G1, G2, G3)):
        np.testing.assert_array_equal(a, b)


def test_one_chunk_is_gd_for_any_beta():
    w = case(T=5, chunk=8)
    args = (w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, w.chunk)
    y, F1, F2, F3, M = O.lact_swiglu_momentum(*args, 0.9)
    yg, G1, G2, G3 = O.lact_swiglu(*args, O.UPDATE_GD, 1)
    np.testing.assert_array_equal(y, yg)
    np.testing.assert_array_equal(F1, G1)


def test_silent_chunks_keep_moving_with_decaying_steps():
    """With eta = 0 after the first chunk, the later chunk gradients vanish, so
    chunk c >= 1 moves each matrix by beta^c G_0 (then renormalises)."""
    beta, chunk = 0.7, 4
    w = case(T=12, chunk=chunk)
    eta = w.eta.copy()
    eta[:, :, chunk:] = 0.0
    _, F1, F2, F3, M = O.lact_swiglu_momentum(w.q, w.k, w.v, eta, w.W1, w.W2, w.W3, chunk, beta)
    for h in range(w.H):
        W = [w.W1[h], w.W2[h], w.W3[h]]
        rho = [O.row_norms(x) for x in W]
        g0 = O.lact_grads(*W, w.k[0, h, :chunk], w.v[0, h, :chunk], w.eta[0, h, :chunk])
        for c in range(3):
            W = [O.renorm_rows(W[i] - beta ** c * g0[i], rho[i]) for i in range(3)]
        for got, want in zip((F1[0, h], F2[0, h], F3[0, h]), W):
            np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)
        for i in range(3):
            np.testing.assert_allclose(M[i][0, h], beta ** 2 * g0[i], rtol=1e-13, atol=1e-16)


def test_unrolled_momentum_sum():
    """Each step moves W by sum_j beta^(c-j) G_j, with G_j the gradient at the
    weights before chunk j (taken from runs on the sequence's prefixes)."""
    beta, chunk, T = 0.5, 4, 16
    w = case(T=T, chunk=chunk, seed=8)
    pre = lambda x, n: x[:, :, :n]
    Wc = [[w.W1[None], w.W2[None], w.W3[None]]]
    for c in range(1, T // chunk + 1):
        _, A1, A2, A3, _ = O.lact_swiglu_momentum(pre(w.q, c * chunk), pre(w.k, c * chunk),
                                                  pre(w.v, c * chunk), pre(w.eta, c * chunk),
                                                  w.W1, w.W2, w.W3, chunk, beta)
        Wc.append([A1, A2, A3])
    for h in range(w.H):
        rho = [O.row_norms(x[0, h]) for x in Wc[0]]
        G = [O.lact_grads(*(x[0, h] for x in Wc[j]), w.k[0, h, j * chunk:(j + 1) * chunk],
                          w.v[0, h, j * chunk:(j + 1) * chunk], w.eta[0, h, j * chunk:(j + 1) * chunk])
             for j in range(T // chunk)]
        for c in range(T // chunk):
            for i in range(3):
                step = sum(beta ** (c - j) * G[j][i] for j in range(c + 1))
                want = O.renorm_rows(Wc[c][i][0, h] - step, rho[i])
                np.testing.assert_allclose(Wc[c + 1][i][0, h], want, rtol=1e-12, atol=1e-14)


def test_resume_with_weights_and_momentum():
    beta, chunk = 0.8, 4
    w = case(T=16, chunk=chunk, seed=5)
    args = (w.W1, w.W2, w.W3, chunk, beta)
    y, F1, F2, F3, M = O.lact_swiglu_momentum(w.q, w.k, w.v, w.eta, *args)
    s = 8
    ya, A1, A2, A3, Ma = O.lact_swiglu_momentum(w.q[:, :, :s], w.k[:, :, :s], w.v[:, :, :s],
                                                w.eta[:, :, :s], *args)
    yb, B1, B2, B3, Mb = O.lact_swiglu_momentum(w.q[:, :, s:], w.k[:, :, s:], w.v[:, :, s:],
                                                w.eta[:, :, s:], A1, A2, A3, chunk, beta, M0=Ma)
    np.testing.assert_allclose(np.concatenate([ya, yb], axis=2), y, rtol=1e-12, atol=1e-13)
    for a, b in zip((B1, B2, B3) + tuple(Mb), (F1, F2, F3) + tuple(M)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_first_chunk_output_depends_on_initial_weights_only():
    w = case(T=12, chunk=4)
    y, *_ = O.lact_swiglu_momentum(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, 4, 0.9)
    k2 = w.k.copy()
    k2[:, :, 4:] += 0.5
    y2, *_ = O.lact_swiglu_momentum(w.q, k2, w.v, w.eta, w.W1, w.W2, w.W3, 4, 0.9)
    np.testing.assert_array_equal(y[:, :, :4], y2[:, :, :4])
    assert np.abs(y[:, :, 8:] - y2[:, :, 8:]).max() > 1e-9
