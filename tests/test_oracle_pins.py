"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test ties an oracle function to something other than itself: a closed
form, an invariant, a special case that reduces to a textbook formula or a
library routine (numpy SVD, torch autograd), finite differences, or a value
table printed on the pages (tests/golden). CPU only.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(B, H, T, dk, dv, seed, eta_scale=0.1, batched_w0=False, w0_std=0.3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk)) / np.sqrt(dk)
    v = rng.standard_normal((B, H, T, dv))
    eta = eta_scale * (0.5 + rng.random((B, H, T)))
    W0 = rng.standard_normal((B, H, dk, dv) if batched_w0 else (H, dk, dv)) * w0_std
    return q, k, v, eta, W0


def relerr(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --------------------------------------------------------------------------
# TTT-Linear
# --------------------------------------------------------------------------

@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_chunk_one_is_the_token_recurrence(loss):
    """Mini-batch GD with b = 1 is the one-step-per-token rule of the TTT
    definition (t' = t for every t)."""
    q, k, v, eta, W0 = rand_case(2, 3, 23, 5, 4, seed=1)
    y1, W1 = O.ttt_linear_minibatch(q, k, v, eta, W0, 1, loss)
    y2, W2 = O.ttt_linear_token_recurrence(q, k, v, eta, W0, loss)
    assert relerr(y1, y2) < 1e-12 and relerr(W1, W2) < 1e-12


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
@pytest.mark.parametrize("b", [1, 2, 5, 16])
@pytest.mark.parametrize("T", [1, 7, 16, 17, 40])
def test_dual_form_equals_minibatch_definition(loss, b, T):
    """The dual form (tril(QK^T) N acting on the chunk-start errors) is an
    exact rewrite of the per-token mini-batch definition, partial chunks too."""
    for batched in (False, True):
        q, k, v, eta, W0 = rand_case(2, 2, T, 6, 5, seed=T * 31 + b, batched_w0=batched)
        y1, W1 = O.ttt_linear_minibatch(q, k, v, eta, W0, b, loss)
        y2, W2 = O.ttt_linear_dual(q, k, v, eta, W0, b, loss)
        assert relerr(y2, y1) < 1e-12 and relerr(W2, W1) < 1e-12


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_loss_gradient_matches_finite_differences(loss):
    """Central differences of the scalar loss (1/2||kW-v||^2 or -(kW).v)."""
    rng = np.random.default_rng(7)
    W = rng.standard_normal((4, 3))
    k = rng.standard_normal(4)
    v = rng.standard_normal(3)
    g = O.loss_grad(W, k, v, loss)
    h = 1e-5
    fd = np.zeros_like(W)
    for a in range(4):
        for c in range(3):
            Wp, Wm = W.copy(), W.copy()
            Wp[a, c] += h
            Wm[a, c] -= h
            fd[a, c] = (O.loss_value(Wp, k, v, loss) - O.loss_value(Wm, k, v, loss)) / (2 * h)
    assert relerr(g, fd) < 1e-8


def test_loss_gradient_matches_autograd():
    """torch autograd (fp64) of the scalar MSE loss as an independent
    differentiation of the same loss."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(8)
    W = rng.standard_normal((5, 4))
    k = rng.standard_normal(5)
    v = rng.standard_normal(4)
    Wt = torch.tensor(W, requires_grad=True)
    L = 0.5 * ((torch.tensor(k) @ Wt - torch.tensor(v)) ** 2).sum()
    L.backward()
    assert relerr(O.loss_grad(W, k, v, O.LOSS_MSE), Wt.grad.numpy()) < 1e-13


def test_deltanet_expansion_and_perfect_binding():
    """MSE step = forgetting + inserting: W - eta k^T(kW - v) =
    W - eta k^T k W + eta k^T v. With ||k|| = 1 and eta = 1 the updated
    weights map k exactly onto v, so querying with q = k returns v."""
    rng = np.random.default_rng(3)
    dk, dv = 8, 6
    W = rng.standard_normal((dk, dv))
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(dv)
    eta = 0.37
    step = W - eta * O.loss_grad(W, k, v, O.LOSS_MSE)
    expanded = W - eta * np.outer(k, k) @ W + eta * np.outer(k, v)
    assert relerr(step, expanded) < 1e-13
    # perfect binding through the oracle's layer function (T=1, chunk=1)
    q = k[None, None, None, :]
    y, Wf = O.ttt_linear_minibatch(q, q, v[None, None, None, :], np.ones((1, 1, 1)),
                                   W[None], 1, O.LOSS_MSE)
    assert relerr(y[0, 0, 0], v) < 1e-13
    assert relerr(k @ Wf[0, 0], v) < 1e-13


def test_mse_step_descends():
    """A small step along -grad lowers the token's loss (sign of the update)."""
    rng = np.random.default_rng(4)
    W = rng.standard_normal((6, 5))
    k, v = rng.standard_normal(6), rng.standard_normal(5)
    _, Wf = O.ttt_linear_minibatch(k[None, None, None], k[None, None, None], v[None, None, None],
                                   np.full((1, 1, 1), 1e-3), W[None], 1, O.LOSS_MSE)
    assert O.loss_value(Wf[0, 0], k, v, O.LOSS_MSE) < O.loss_value(W, k, v, O.LOSS_MSE)


@pytest.mark.parametrize("b", [1, 3, 16, 64])
def test_inner_product_loss_is_causal_linear_attention(b):
    """Inner-product loss with constant eta and W0 = 0 gives
    y_t = eta * sum_{i<=t} (q_t . k_i) v_i, the softmax-free attention form,
    for every chunk size (its gradient does not depend on W)."""
    rng = np.random.default_rng(11)
    B, H, T, dk, dv = 1, 2, 37, 5, 3
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    eta = np.full((B, H, T), 0.25)
    y, S = O.ttt_linear_minibatch(q, k, v, eta, np.zeros((H, dk, dv)), b, O.LOSS_NEG_DOT)
    ref = np.zeros_like(y)
    for h in range(H):
        for t in range(T):
            for i in range(t + 1):
                ref[0, h, t] += 0.25 * float(q[0, h, t] @ k[0, h, i]) * v[0, h, i]
    assert relerr(y, ref) < 1e-12
    y_la, S_la = O.linear_attention(q, k, v, eta, np.zeros((H, dk, dv)))
    assert relerr(y_la, ref) < 1e-12 and relerr(S, S_la) < 1e-12
    yd, _ = O.ttt_linear_dual(q, k, v, eta, np.zeros((H, dk, dv)), b, O.LOSS_NEG_DOT)
    assert relerr(yd, ref) < 1e-12


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_zero_learning_rate_is_a_fixed_linear_map(loss):
    q, k, v, _, W0 = rand_case(2, 2, 19, 4, 3, seed=5)
    eta = np.zeros((2, 2, 19))
    for fn in (O.ttt_linear_minibatch, O.ttt_linear_dual):
        y, Wf = fn(q, k, v, eta, W0, 4, loss)
        assert np.array_equal(Wf, np.broadcast_to(W0, Wf.shape))
        assert relerr(y, np.einsum("bhta,hac->bhtc", q, W0)) < 1e-13


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_resume_from_final_state(loss):
    """Splitting the sequence at a chunk boundary and feeding W_final back as
    W0 reproduces the whole run (mini-batch rule: only W crosses chunks)."""
    q, k, v, eta, W0 = rand_case(2, 2, 45, 4, 5, seed=9)
    y, Wf = O.ttt_linear_dual(q, k, v, eta, W0, 8, loss)
    ya, Wa = O.ttt_linear_dual(q[:, :, :16], k[:, :, :16], v[:, :, :16], eta[:, :, :16], W0, 8, loss)
    yb, Wb = O.ttt_linear_dual(q[:, :, 16:], k[:, :, 16:], v[:, :, 16:], eta[:, :, 16:], Wa, 8, loss)
    assert relerr(np.concatenate([ya, yb], axis=2), y) < 1e-12 and relerr(Wb, Wf) < 1e-12


def test_arithmetic_intensity_formula_and_table():
    """r = 2h^2b/(2h^2+4hb) = b/(1+2b/h) <= min(h/2, b); the page's table
    lists the bound min(h/2, b) (tests/golden/arithmetic_intensity_table.json)."""
    with open(os.path.join(GOLDEN, "arithmetic_intensity_table.json")) as f:
        table = json.load(f)
    h = table["h_for_check"]
    for b in (1, 16, 64, 256, 2048, 8192):
        for hh in (64, 128, 256, h):
            r = O.arithmetic_intensity(b, hh)
            assert abs(r - b / (1 + 2 * b / hh)) < 1e-9 * r
            assert r <= min(hh / 2, b) + 1e-9
    for row in table["rows"]:
        bound = min(h / 2, row["chunk"])
        expect = h / 2 if row["approx"] == "h/2" else row["approx"]
        assert bound == expect


# --------------------------------------------------------------------------
# LaCT SwiGLU
# --------------------------------------------------------------------------

def lact_case(n=5, dk=3, dv=3, dh=4, seed=0):
    rng = np.random.default_rng(seed)
    W1 = rng.standard_normal((dh, dk))
    W2 = rng.standard_normal((dv, dh))
    W3 = rng.standard_normal((dh, dk))
    K = rng.standard_normal((n, dk))
    V = rng.standard_normal((n, dv))
    eta = 0.1 + rng.random(n)
    return W1, W2, W3, K, V, eta


def test_swiglu_silu_branch_special_cases():
    """silu(z) -> z for z >> 0 and -> 0 for z << 0, so with W1 x large
    positive f(x) -> W2 ((W1 x) * (W3 x)) and with W1 x large negative
    f(x) -> 0: this fixes which of W1, W3 passes through the SiLU."""
    x = np.array([[1.0]])
    W2 = np.array([[3.0]])
    f_pos = O.swiglu(np.array([[60.0]]), W2, np.array([[-2.0]]), x)
    assert abs(f_pos[0, 0] - 3.0 * 60.0 * -2.0) < 1e-9
    f_neg = O.swiglu(np.array([[-60.0]]), W2, np.array([[5.0]]), x)
    assert abs(f_neg[0, 0]) < 1e-20
    # silu(0) = 0 and silu'(0) = 1/2
    assert O.silu(0.0) == 0.0 and O.silu_grad(0.0) == 0.5


def test_swiglu_gradients_match_finite_differences():
    W1, W2, W3, K, V, eta = lact_case()
    G = O.lact_grads(W1, W2, W3, K, V, eta)
    h = 1e-6
    for idx, W in enumerate((W1, W2, W3)):
        fd = np.zeros_like(W)
        for r in range(W.shape[0]):
            for c in range(W.shape[1]):
                Ws_p = [W1.copy(), W2.copy(), W3.copy()]
                Ws_m = [W1.copy(), W2.copy(), W3.copy()]
                Ws_p[idx][r, c] += h
                Ws_m[idx][r, c] -= h
                fd[r, c] = (O.lact_loss(*Ws_p, K, V, eta) - O.lact_loss(*Ws_m, K, V, eta)) / (2 * h)
        assert relerr(G[idx], fd) < 1e-7, idx


def test_swiglu_gradients_match_autograd():
    torch = pytest.importorskip("torch")
    W1, W2, W3, K, V, eta = lact_case(n=9, dk=6, dv=5, dh=7, seed=2)
    t = [torch.tensor(W, requires_grad=True) for W in (W1, W2, W3)]
    Kt, Vt, et = map(torch.tensor, (K, V, eta))
    f = (torch.nn.functional.silu(Kt @ t[0].T) * (Kt @ t[2].T)) @ t[1].T
    L = -(et[:, None] * f * Vt).sum()
    L.backward()
    G = O.lact_grads(W1, W2, W3, K, V, eta)
    for g, tt in zip(G, t):
        assert relerr(g, tt.grad.numpy()) < 1e-12


def test_lact_gd_step_raises_inner_product():
    """A small GD step on -f(k).v increases f(k).v (sign of the update)."""
    W1, W2, W3, K, V, eta = lact_case(n=1, seed=4)
    G1, G2, G3 = O.lact_grads(W1, W2, W3, K, V, 1e-4 * eta)
    before = float(O.swiglu(W1, W2, W3, K) @ V[0])
    after = float(O.swiglu(W1 - G1, W2 - G2, W3 - G3, K) @ V[0])
    assert after > before


@pytest.mark.parametrize("shape", [(12, 5), (5, 12), (7, 7)])
def test_newton_schulz_matches_svd_polynomial(shape):
    """NS5(G) = U p5(S / (||G||_F + eps)) V^T, with p(s) = a s + b s^3 + c s^5
    applied five times, from numpy.linalg.svd."""
    rng = np.random.default_rng(sum(shape))
    G = rng.standard_normal(shape) * 0.01
    U, S, Vt = np.linalg.svd(G, full_matrices=False)
    s = S / (np.linalg.norm(G) + O.NS_EPS)
    a, b, c = O.NS_COEFFS
    for _ in range(O.NS_STEPS):
        s = a * s + b * s ** 3 + c * s ** 5
    ref = (U * s) @ Vt
    assert relerr(O.newton_schulz5(G), ref) < 1e-10
    # the quintic pushes singular values of a well-conditioned G towards 1
    sv = np.linalg.svd(O.newton_schulz5(G), compute_uv=False)
    assert sv.max() < 1.25


def test_renorm_rows_restores_norms_and_keeps_zero_rows():
    rng = np.random.default_rng(6)
    W = rng.standard_normal((5, 4))
    W[2] = 0.0
    rho = np.array([1.0, 2.0, 3.0, 0.5, 4.0])
    R = O.renorm_rows(W, rho)
    n = O.row_norms(R)
    assert np.allclose(n[[0, 1, 3, 4]], rho[[0, 1, 3, 4]], rtol=1e-14)
    assert np.all(R[2] == 0.0)
    # direction of each row is kept
    assert np.allclose(R[0] / n[0], W[0] / np.linalg.norm(W[0]))


def tiny_lact(T=23, chunk=6, seed=3, rule=O.UPDATE_GD, B=2, H=2, d=4, dh=6):
    w = synth.make_lact(B, H, T, d, dh, chunk, rule, seed, dtype=synth.F32, eta_scale=0.05)
    return w


@pytest.mark.parametrize("rule", [O.UPDATE_GD, O.UPDATE_MUON])
def test_lact_renorm_invariant_and_resume(rule):
    w = tiny_lact(rule=rule)
    args = (w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3)
    y, F1, F2, F3 = O.lact_swiglu(*args, w.chunk, rule, 1)
    for F, W0 in ((F1, w.W1), (F2, w.W2), (F3, w.W3)):
        assert np.allclose(O.row_norms(F), np.broadcast_to(O.row_norms(W0), O.row_norms(F).shape),
                           rtol=1e-12)
    # resume: split at 12 (a multiple of chunk) and chain the final weights
    s = 12
    ya, A1, A2, A3 = O.lact_swiglu(w.q[:, :, :s], w.k[:, :, :s], w.v[:, :, :s], w.eta[:, :, :s],
                                   w.W1, w.W2, w.W3, w.chunk, rule, 1)
    yb, B1, B2, B3 = O.lact_swiglu(w.q[:, :, s:], w.k[:, :, s:], w.v[:, :, s:], w.eta[:, :, s:],
                                   A1, A2, A3, w.chunk, rule, 1)
    assert relerr(np.concatenate([ya, yb], axis=2), y) < 1e-10
    assert relerr(B2, F2) < 1e-10


def test_lact_apply_then_update_causality():
    """Causal order: chunk c's outputs use only chunks < c for the weights,
    so perturbing k, v or eta of chunk c (or later) leaves every output up to
    and including chunk c bit-identical; chunk 0 depends on W0 and Q0 only."""
    w = tiny_lact(T=24, chunk=6)
    args = [w.q, w.k, w.v, w.eta]
    y, *_ = O.lact_swiglu(*args, w.W1, w.W2, w.W3, w.chunk, O.UPDATE_GD, 1)
    y0 = O.swiglu(w.W1[0], w.W2[0], w.W3[0], w.q[0, 0, :6])
    assert np.array_equal(y[0, 0, :6], y0)
    for c in range(4):
        s = c * 6
        for which in (1, 2, 3):
            pert = [a.copy() for a in args]
            pert[which][:, :, s:s + 6] *= 1.5
            yp, *_ = O.lact_swiglu(*pert, w.W1, w.W2, w.W3, w.chunk, O.UPDATE_GD, 1)
            assert np.array_equal(yp[:, :, :s + 6], y[:, :, :s + 6])
            if c < 3:
                assert not np.allclose(yp[:, :, s + 6:], y[:, :, s + 6:])


def test_lact_non_causal_updates_before_apply():
    """causal=0 (update, then apply): chunk c's own keys move its outputs, and
    chunk 0's output is f with the once-updated weights."""
    w = tiny_lact(T=12, chunk=6)
    args = [w.q, w.k, w.v, w.eta]
    y, *_ = O.lact_swiglu(*args, w.W1, w.W2, w.W3, w.chunk, O.UPDATE_GD, 0)
    pert = [a.copy() for a in args]
    pert[1][:, :, :6] *= 1.5
    yp, *_ = O.lact_swiglu(*pert, w.W1, w.W2, w.W3, w.chunk, O.UPDATE_GD, 0)
    assert not np.allclose(yp[:, :, :6], y[:, :, :6])
    g1, g2, g3 = O.lact_grads(w.W1[0], w.W2[0], w.W3[0], w.k[0, 0, :6], w.v[0, 0, :6], w.eta[0, 0, :6])
    n1, n2, n3 = (O.renorm_rows(W - g, O.row_norms(W)) for W, g in
                  ((w.W1[0], g1), (w.W2[0], g2), (w.W3[0], g3)))
    assert relerr(y[0, 0, :6], O.swiglu(n1, n2, n3, w.q[0, 0, :6])) < 1e-13


def test_lact_zero_learning_rate():
    """eta = 0: G = 0 (and NS5 of a zero matrix is zero), renorm of unchanged
    rows is the identity, so y = f_{W0}(q) and the weights stay W0."""
    for rule in (O.UPDATE_GD, O.UPDATE_MUON):
        w = tiny_lact(T=13, chunk=4, rule=rule)
        eta = np.zeros_like(w.eta)
        for causal in (0, 1):
            y, F1, F2, F3 = O.lact_swiglu(w.q, w.k, w.v, eta, w.W1, w.W2, w.W3, 4, rule, causal)
            ref = np.stack([np.stack([O.swiglu(w.W1[h], w.W2[h], w.W3[h], w.q[b, h])
                                      for h in range(w.H)]) for b in range(w.B)])
            assert relerr(y, ref) < 1e-14
            assert relerr(F1, np.broadcast_to(w.W1, F1.shape)) < 1e-14


def test_lact_prefix_matches_full_run():
    w = tiny_lact(T=30, chunk=6)
    y, *_ = O.lact_swiglu(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, 6, O.UPDATE_GD, 1)
    yp = O.lact_swiglu_prefix(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, 6, O.UPDATE_GD, 2, (1, 1))
    assert np.array_equal(yp, y[1, 1, :12])


# --------------------------------------------------------------------------
# Stored regression values (written by tests/golden/make_golden.py, which
# calls only oracle/ and the seeded input generator).
# --------------------------------------------------------------------------

def test_oracle_matches_stored_golden_values():
    from tests.golden.make_golden import CASES, compute
    with open(os.path.join(GOLDEN, "oracle_small_cases.json")) as f:
        stored = json.load(f)
    for name in CASES:
        got = compute(name)
        for key, val in stored[name].items():
            assert np.allclose(np.asarray(got[key]), np.asarray(val), rtol=1e-12, atol=1e-14), (name, key)


# --------------------------------------------------------------------------
# The Muon branch of the LaCT scan, composed by hand from pinned pieces:
# lact_grads (finite differences), the Newton-Schulz polynomial evaluated on
# numpy's SVD, and the row renorm written out as a scale per row.
# ("Test-Time Training Done Right" review 3.3: the summed gradient is
# orthogonalised by Newton-Schulz, then the step, then L2 normalisation.)
# --------------------------------------------------------------------------

def _ns5_by_svd(G):
    U, S, Vt = np.linalg.svd(G, full_matrices=False)
    s = S / (np.sqrt(np.sum(G * G)) + 1e-7)
    a, b, c = 3.4445, -4.7750, 2.0315
    for _ in range(5):
        s = a * s + b * s ** 3 + c * s ** 5
    return (U * s) @ Vt


def _rescale_rows(W, W_init):
    target = np.sqrt(np.sum(W_init * W_init, axis=1))
    return W * (target / np.sqrt(np.sum(W * W, axis=1)))[:, None]


def _swiglu_by_hand(W1, W2, W3, X):
    h1 = X @ W1.T
    return ((h1 / (1.0 + np.exp(-h1))) * (X @ W3.T)) @ W2.T


def _muon_chunk_by_hand(Ws, W_init, K, V, eta):
    G = O.lact_grads(*Ws, K, V, eta)
    return [_rescale_rows(W - _ns5_by_svd(g), Wi) for W, g, Wi in zip(Ws, G, W_init)]


@pytest.mark.parametrize("causal", [1, 0])
def test_lact_muon_scan_is_svd_polynomial_step_then_renorm(causal):
    """Two chunks (the second ragged) of one (batch, head) under Muon: the
    weights after each chunk are renorm(W - U p5(S/(||G||_F+eps)) V^T) with G
    taken at the renormalised weights of the previous chunk, and the outputs
    are f of the weights before (causal) or after (non-causal) the chunk's
    update. A scan that skipped Newton-Schulz, used the raw weights for the
    second gradient, or renormalised to the previous chunk's norms fails."""
    w = synth.make_lact(1, 1, 11, 3, 5, 6, O.UPDATE_MUON, 21, dtype=synth.F32, eta_scale=0.2)
    q, k, v, eta = (np.float64(x[0, 0]) for x in (w.q, w.k, w.v, w.eta))
    W_init = [np.float64(W[0]) for W in (w.W1, w.W2, w.W3)]
    y, F1, F2, F3 = O.lact_swiglu(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, 6, O.UPDATE_MUON, causal)
    W_a = _muon_chunk_by_hand(W_init, W_init, k[:6], v[:6], eta[:6])
    W_b = _muon_chunk_by_hand(W_a, W_init, k[6:], v[6:], eta[6:])
    for F, ref in zip((F1, F2, F3), W_b):
        assert relerr(F[0, 0], ref) < 1e-10
    y_ref = np.concatenate([_swiglu_by_hand(*(W_init if causal else W_a), q[:6]),
                            _swiglu_by_hand(*(W_a if causal else W_b), q[6:])])
    assert relerr(y[0, 0], y_ref) < 1e-10
    # the step is not a plain gradient step: Newton-Schulz changed the weights
    W_gd = [_rescale_rows(W - g, Wi) for W, g, Wi in
            zip(W_init, O.lact_grads(*W_init, k[:6], v[:6], eta[:6]), W_init)]
    assert max(relerr(a, b) for a, b in zip(W_a, W_gd)) > 1e-3
