"""The 64-token group form used by the d = 64 MSE kernel equals the mini-batch
definition (fp64, CPU).

Within a group that starts with weights W_g, sub-block c (16 tokens) has
    E_c = K_c W_s - V_c - sum_{c' < c, c' in an earlier chunk} K_c K_c'^T N_c' E_c'
(W_s: start weights of the chunk open at the group start), and
    y_t = q_t W_g - sum_{i <= t in the group} eta_i (q_t . k_i) e_i,
    W_{g+1} = W_g - sum_{i in the group} eta_i k_i^T e_i.
This restates that algebra in numpy and compares it with the oracle's
definition for every chunk size the kernel accepts, including ragged ends.
"""
import numpy as np
import pytest

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import synth

G, S = 64, 16


def group_form(q, k, v, eta, W0, chunk):
    T = q.shape[0]
    W = W0.copy()
    Ws = W0.copy()
    y = np.zeros((T, W0.shape[1]))
    for g0 in range(0, T, G):
        subs = [(a, min(a + S, T)) for a in range(g0, min(g0 + G, T), S)]
        E = []
        for c, (a, b) in enumerate(subs):
            e = k[a:b] @ Ws - v[a:b]
            for cp in range(c):
                ap, bp = subs[cp]
                if ap // chunk == a // chunk:
                    continue
                e = e - (k[a:b] @ k[ap:bp].T) @ (eta[ap:bp, None] * E[cp])
            E.append(e)
        n = sum(b - a for a, b in subs)
        Eg, kg, qg, eg = np.concatenate(E), k[g0:g0 + n], q[g0:g0 + n], eta[g0:g0 + n]
        P = np.tril(qg @ kg.T) * eg[None, :]
        y[g0:g0 + n] = qg @ W - P @ Eg
        W = W - kg.T @ (eg[:, None] * Eg)
        if (g0 + G) % chunk == 0:
            Ws = W.copy()
    return y, W


@pytest.mark.parametrize("chunk", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("T", [256, 200, 77, 1])
def test_group_form_equals_definition(chunk, T):
    w = synth.make_ttt_linear(1, 1, T, 64, 64, chunk, synth.F32, synth.LOSS_MSE,
                              seed=chunk + T, eta_kind="softplus", eta_scale=0.5)
    f = lambda n: w.f64(n)[0, 0]
    y, W = group_form(f("q"), f("k"), f("v"), f("eta"), w.f64("W0")[0], chunk)
    yo, Wo = O.ttt_linear_minibatch(w.q, w.k, w.v, w.eta, w.W0, chunk, O.LOSS_MSE)
    assert np.abs(y - yo[0, 0]).max() <= 1e-12 * max(1.0, np.abs(yo).max())
    assert np.abs(W - Wo[0, 0]).max() <= 1e-12 * max(1.0, np.abs(Wo).max())


def test_group_form_needs_the_correction_terms():
    """Dropping the cross-chunk corrections (chunk 16) changes the result: the
    identity above is not vacuous."""
    w = synth.make_ttt_linear(1, 1, 128, 64, 64, 16, synth.F32, synth.LOSS_MSE, seed=3,
                              eta_kind="softplus", eta_scale=0.5)
    f = lambda n: w.f64(n)[0, 0]
    y, _ = group_form(f("q"), f("k"), f("v"), f("eta"), w.f64("W0")[0], 10 ** 9)
    yo, _ = O.ttt_linear_minibatch(w.q, w.k, w.v, w.eta, w.W0, 16, O.LOSS_MSE)
    assert np.abs(y - yo[0, 0]).max() > 1e-3
