"""Pins of the backward-pass oracles (training).

``ttt_linear_minibatch_bwd`` (the TTT-Linear reverse chunk scan) and
``lact_backward.lact_swiglu_bwd`` (the LaCT layer) are checked against things
other than themselves: central finite differences of the pinned forward
definitions (``ttt_linear_minibatch``, ``lact_swiglu``) along random
directions, the closed forms of the zero-learning-rate case, the
batch-sharing invariant of dW0, and (LaCT) equality of the restated forward
with the numpy oracle. CPU only.
"""
import numpy as np
import pytest

from oracle import ttt_oracle as O


def case(B, H, T, dk, dv, seed, batched_w0=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk)) / np.sqrt(dk)
    v = rng.standard_normal((B, H, T, dv))
    eta = 0.2 * (0.5 + rng.random((B, H, T)))
    W0 = 0.3 * rng.standard_normal((B, H, dk, dv) if batched_w0 else (H, dk, dv))
    dy = rng.standard_normal((B, H, T, dv))
    dWf = rng.standard_normal((B, H, dk, dv))
    return rng, (q, k, v, eta, W0), dy, dWf


def objective(args, chunk, loss, dy, dWf):
    y, W = O.ttt_linear_minibatch(*args, chunk, loss)
    return float(np.sum(y * dy) + (np.sum(W * dWf) if dWf is not None else 0.0))


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
@pytest.mark.parametrize("chunk", [1, 3, 4, 10])
@pytest.mark.parametrize("batched_w0", [False, True])
def test_gradients_match_finite_differences(loss, chunk, batched_w0):
    """<grad, d> equals (L(x + h d) - L(x - h d)) / 2h for every input; T = 10
    gives a ragged last chunk for chunk 3 and 4."""
    rng, args, dy, dWf = case(2, 2, 10, 4, 5, seed=chunk * 10 + loss + 3 * batched_w0,
                              batched_w0=batched_w0)
    grads = O.ttt_linear_minibatch_bwd(*args, chunk, loss, dy, dWf)
    h = 1e-5
    for n, name in enumerate(("q", "k", "v", "eta", "W0")):
        d = rng.standard_normal(args[n].shape)
        plus = list(args)
        minus = list(args)
        plus[n] = args[n] + h * d
        minus[n] = args[n] - h * d
        fd = (objective(plus, chunk, loss, dy, dWf) - objective(minus, chunk, loss, dy, dWf)) / (2 * h)
        an = float(np.sum(grads[n] * d))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, fd, an)


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_without_final_state_gradient(loss):
    """dW_final = None is the objective sum(y * dy) alone."""
    rng, args, dy, _ = case(1, 2, 9, 3, 4, seed=21)
    grads = O.ttt_linear_minibatch_bwd(*args, 4, loss, dy, None)
    h = 1e-5
    for n in range(5):
        d = rng.standard_normal(args[n].shape)
        plus = list(args)
        minus = list(args)
        plus[n] = args[n] + h * d
        minus[n] = args[n] - h * d
        fd = (objective(plus, 4, loss, dy, None) - objective(minus, 4, loss, dy, None)) / (2 * h)
        assert abs(fd - float(np.sum(grads[n] * d))) <= 1e-7 * max(1.0, abs(fd))


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_zero_learning_rate_closed_form(loss):
    """With eta = 0 the layer is y_t = q_t W0 and W_final = W0, so
    dq_t = dy_t W0^T, dk = dv = 0 and dW0 = sum_t q_t^T dy_t + dW_final
    (summed over the batch for a shared W0)."""
    _, (q, k, v, eta, W0), dy, dWf = case(2, 3, 8, 4, 6, seed=5)
    eta = np.zeros_like(eta)
    dq, dk, dv, deta, dW0 = O.ttt_linear_minibatch_bwd(q, k, v, eta, W0, 3, loss, dy, dWf)
    np.testing.assert_allclose(dq, np.einsum("bhtc,hac->bhta", dy, W0), rtol=1e-12, atol=1e-12)
    assert np.all(dk == 0) and np.all(dv == 0)
    want = np.einsum("bhta,bhtc->hac", q, dy) + dWf.sum(axis=0)
    np.testing.assert_allclose(dW0, want, rtol=1e-12, atol=1e-12)
    # the learning-rate gradient is the only one that sees the update
    assert np.any(deta != 0)


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_shared_w0_gradient_is_the_batch_sum(loss):
    """A W0 shared by the batch gets the sum of the per-sequence gradients
    that the same W0 copied per sequence receives."""
    _, (q, k, v, eta, W0), dy, dWf = case(3, 2, 7, 4, 4, seed=9)
    shared = O.ttt_linear_minibatch_bwd(q, k, v, eta, W0, 2, loss, dy, dWf)
    per_seq = O.ttt_linear_minibatch_bwd(q, k, v, eta, np.broadcast_to(W0, (3,) + W0.shape).copy(),
                                         2, loss, dy, dWf)
    for a, b in zip(shared[:4], per_seq[:4]):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(shared[4], per_seq[4].sum(axis=0), rtol=1e-12, atol=1e-12)


def test_inner_product_gradient_does_not_depend_on_v():
    """The inner-product layer is linear in v (y and W_final are), so its
    gradient with respect to v does not change when v does."""
    _, (q, k, v, eta, W0), dy, dWf = case(1, 2, 8, 4, 4, seed=13)
    a = O.ttt_linear_minibatch_bwd(q, k, v, eta, W0, 3, O.LOSS_NEG_DOT, dy, dWf)
    b = O.ttt_linear_minibatch_bwd(q, k, 2.0 * v + 1.0, eta, W0, 3, O.LOSS_NEG_DOT, dy, dWf)
    np.testing.assert_allclose(a[2], b[2], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# LaCT backward (oracle/lact_backward.py)
# --------------------------------------------------------------------------

from oracle import lact_backward as LB  # noqa: E402


def lact_case(B, H, T, dk, dv, dh, seed, shared=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    eta = 0.3 * (0.5 + rng.random((B, H, T)))
    lead = (H,) if shared else (B, H)
    W1 = rng.standard_normal(lead + (dh, dk)) / np.sqrt(dk)
    W2 = rng.standard_normal(lead + (dv, dh)) / np.sqrt(dh)
    W3 = rng.standard_normal(lead + (dh, dk)) / np.sqrt(dk)
    dy = rng.standard_normal((B, H, T, dv))
    dWf = (rng.standard_normal((B, H, dh, dk)), rng.standard_normal((B, H, dv, dh)),
           rng.standard_normal((B, H, dh, dk)))
    return rng, [q, k, v, eta, W1, W2, W3], dy, dWf


def lact_objective(args, chunk, rule, causal, dy, dWf):
    y, F1, F2, F3 = O.lact_swiglu(*args, chunk, rule, causal)
    return float(np.sum(y * dy) + sum(np.sum(F * d) for F, d in zip((F1, F2, F3), dWf)))


@pytest.mark.parametrize("rule", [O.UPDATE_GD, O.UPDATE_MUON])
@pytest.mark.parametrize("causal", [1, 0])
def test_lact_torch_forward_equals_the_oracle(rule, causal):
    _, args, _, _ = lact_case(1, 2, 7, 3, 3, 4, seed=1 + rule + 2 * causal)
    y, F1, F2, F3 = O.lact_swiglu(*args, 3, rule, causal)
    for h in range(2):
        t = [LB._t(x[0, h]) for x in args[:4]] + [LB._t(W[h]) for W in args[4:]]
        yt, f1, f2, f3 = LB.lact_swiglu_torch(*t, 3, rule, causal)
        np.testing.assert_allclose(yt.numpy(), y[0, h], rtol=1e-11, atol=1e-12)
        for ft, F in zip((f1, f2, f3), (F1, F2, F3)):
            np.testing.assert_allclose(ft.numpy(), F[0, h], rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("rule,causal,shared", [(O.UPDATE_GD, 1, True), (O.UPDATE_GD, 0, False),
                                                (O.UPDATE_MUON, 1, True), (O.UPDATE_MUON, 0, True)])
def test_lact_gradients_match_finite_differences(rule, causal, shared):
    """Every input, with a ragged last chunk (T = 7, chunk 3)."""
    rng, args, dy, dWf = lact_case(2, 1, 7, 3, 3, 4, seed=11 + rule + 2 * causal, shared=shared)
    grads = LB.lact_swiglu_bwd(*args, 3, rule, causal, dy, dWf)
    h = 1e-6
    for n, name in enumerate(("q", "k", "v", "eta", "W1", "W2", "W3")):
        d = rng.standard_normal(args[n].shape)
        plus = list(args)
        minus = list(args)
        plus[n] = args[n] + h * d
        minus[n] = args[n] - h * d
        fd = (lact_objective(plus, 3, rule, causal, dy, dWf) -
              lact_objective(minus, 3, rule, causal, dy, dWf)) / (2 * h)
        an = float(np.sum(grads[n] * d))
        assert abs(fd - an) <= 2e-6 * max(1.0, abs(fd)), (name, fd, an)


def test_lact_zero_learning_rate_closed_form():
    """With eta = 0 nothing is updated (and the renorm returns the initial
    rows), so y_t = f_W(q_t) = W2 (silu(W1 q_t) * W3 q_t) and the gradients
    are the SwiGLU ones: dk = dv = 0, the final-weight gradients pass to the
    initial weights unchanged."""
    _, args, dy, dWf = lact_case(1, 1, 6, 3, 3, 4, seed=4)
    args[3] = np.zeros_like(args[3])
    dq, dk, dv, _, dW1, dW2, dW3 = LB.lact_swiglu_bwd(*args, 2, O.UPDATE_GD, 1, dy, dWf)
    q, W1, W2, W3 = args[0][0, 0], args[4][0], args[5][0], args[6][0]
    H1, H3 = q @ W1.T, q @ W3.T
    act = O.silu(H1) * H3
    g = dy[0, 0]
    dact = g @ W2
    dH1 = dact * H3 * O.silu_grad(H1)
    dH3 = dact * O.silu(H1)
    np.testing.assert_allclose(dq[0, 0], dH1 @ W1 + dH3 @ W3, rtol=1e-10, atol=1e-12)
    assert np.all(dk == 0) and np.all(dv == 0)
    np.testing.assert_allclose(dW2[0], g.T @ act + dWf[1][0, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dW1[0], dH1.T @ q + dWf[0][0, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dW3[0], dH3.T @ q + dWf[2][0, 0], rtol=1e-10, atol=1e-12)
