"""Pins of the TTT-Linear backward oracle (the reverse chunk scan).

``ttt_linear_minibatch_bwd`` is checked against things other than itself:
central finite differences of the pinned forward definition
(``ttt_linear_minibatch``) along random directions, the closed form of the
zero-learning-rate case, and the batch-sharing invariant of dW0. CPU only.
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
