"""Pins of the TTT-MLP oracle (the scope table's "next" row f3), CPU only.

The pages define the fast weight f(x) = W2 ReLU(W1 x + b1) + b2 and the TTT
framework (self-supervised loss, mini-batch gradient descent) but print no
numbers for it. The readings taken: the loss is the MSE of TTT-Linear,
1/2 ||f(k) - v||^2; all four parameters are fast weights; each chunk uses its
start weights for every gradient and token t sees the updates of tokens
<= t; the ReLU derivative at 0 is 0.
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O


def params(rng, dk, dh, dv, scale=1.0):
    return (scale * rng.standard_normal((dh, dk)) / np.sqrt(dk), 0.1 * rng.standard_normal(dh),
            scale * rng.standard_normal((dv, dh)) / np.sqrt(dh), 0.1 * rng.standard_normal(dv))


def tokens(rng, T, dk, dv):
    return (rng.standard_normal((T, dk)), rng.standard_normal((T, dk)),
            rng.standard_normal((T, dv)), 0.1 * (0.5 + rng.random(T)))


def test_gradients_match_finite_differences():
    rng = np.random.default_rng(1)
    P = params(rng, 3, 5, 4)
    _, k, v, _ = tokens(rng, 1, 3, 4)
    g = O.mlp_grads(*P, k[0], v[0])
    h = 1e-6
    for n in range(4):
        d = rng.standard_normal(P[n].shape)
        plus = list(P)
        minus = list(P)
        plus[n] = P[n] + h * d
        minus[n] = P[n] - h * d
        fd = (O.mlp_loss(*plus, k[0], v[0]) - O.mlp_loss(*minus, k[0], v[0])) / (2 * h)
        assert abs(fd - np.sum(g[n] * d)) <= 1e-6 * max(1.0, abs(fd))


def test_gradients_match_autograd():
    rng = np.random.default_rng(2)
    P = params(rng, 4, 6, 3)
    _, k, v, _ = tokens(rng, 1, 4, 3)
    tP = [torch.tensor(p, dtype=torch.float64, requires_grad=True) for p in P]
    kk, vv = torch.tensor(k[0]), torch.tensor(v[0])
    out = tP[2] @ torch.relu(tP[0] @ kk + tP[1]) + tP[3]
    (0.5 * torch.sum((out - vv) ** 2)).backward()
    for g, t in zip(O.mlp_grads(*P, k[0], v[0]), tP):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_apply_is_the_two_layer_relu_mlp():
    """ReLU on the hidden layer (not the output): a negative hidden unit
    contributes nothing, a positive one passes linearly."""
    W1 = np.array([[1.0, 0.0], [-1.0, 0.0]])
    b1 = np.zeros(2)
    W2 = np.array([[2.0, 3.0]])
    b2 = np.array([0.5])
    x = np.array([[2.0, 7.0], [-2.0, 7.0]])
    np.testing.assert_allclose(O.mlp_apply(W1, b1, W2, b2, x)[:, 0], [4.5, 6.5])


@pytest.mark.parametrize("T", [1, 6, 13])
def test_chunk_one_is_the_token_recurrence(T):
    rng = np.random.default_rng(T)
    P = params(rng, 3, 5, 4)
    q, k, v, eta = tokens(rng, T, 3, 4)
    y1, F1 = O.ttt_mlp_minibatch(q, k, v, eta, *P, 1)
    y2, F2 = O.ttt_mlp_token_recurrence(q, k, v, eta, *P)
    np.testing.assert_allclose(y1, y2, rtol=1e-13, atol=1e-13)
    for a, b in zip(F1, F2):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def test_dead_hidden_layer_reduces_to_a_bias_regression():
    """With every hidden unit inactive (W1 = 0, b1 < 0) only b2 learns, and
    inside a chunk b2_t = b2_s - sum_{i<=t} eta_i (b2_s - v_i)."""
    rng = np.random.default_rng(4)
    T, chunk, dk, dh, dv = 12, 5, 3, 4, 2
    q, k, v, eta = tokens(rng, T, dk, dv)
    W1, b1 = np.zeros((dh, dk)), -np.ones(dh)
    W2, b2 = rng.standard_normal((dv, dh)), rng.standard_normal(dv)
    y, (F1, Fb1, F2, Fb2) = O.ttt_mlp_minibatch(q, k, v, eta, W1, b1, W2, b2, chunk)
    bs = b2.copy()
    for s in range(0, T, chunk):
        start = bs.copy()
        for t in range(s, min(s + chunk, T)):
            bs = start - np.sum(eta[s:t + 1, None] * (start - v[s:t + 1]), axis=0)
            np.testing.assert_allclose(y[t], bs, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Fb2, bs, rtol=1e-12, atol=1e-12)
    assert np.array_equal(F1, W1) and np.array_equal(Fb1, b1) and np.array_equal(F2, W2)


def test_zero_learning_rate_applies_the_initial_mlp():
    rng = np.random.default_rng(5)
    P = params(rng, 3, 5, 4)
    q, k, v, eta = tokens(rng, 8, 3, 4)
    y, F = O.ttt_mlp_minibatch(q, k, v, np.zeros_like(eta), *P, 3)
    np.testing.assert_allclose(y, O.mlp_apply(*P, q), rtol=1e-13, atol=1e-13)
    for a, b in zip(F, P):
        assert np.array_equal(a, b)


def test_a_small_step_lowers_the_chunk_loss():
    rng = np.random.default_rng(6)
    P = params(rng, 4, 8, 4)
    _, k, v, _ = tokens(rng, 16, 4, 4)
    eta = np.full(16, 1e-3)
    before = sum(O.mlp_loss(*P, k[i], v[i]) for i in range(16))
    _, F = O.ttt_mlp_minibatch(k, k, v, eta, *P, 16)
    after = sum(O.mlp_loss(*F, k[i], v[i]) for i in range(16))
    assert after < before


@pytest.mark.parametrize("chunk,split", [(4, 8), (3, 9), (1, 5)])
def test_resume_from_the_final_weights(chunk, split):
    rng = np.random.default_rng(chunk + split)
    P = params(rng, 3, 5, 4)
    q, k, v, eta = tokens(rng, 16, 3, 4)
    y, F = O.ttt_mlp_minibatch(q, k, v, eta, *P, chunk)
    ya, Fa = O.ttt_mlp_minibatch(q[:split], k[:split], v[:split], eta[:split], *P, chunk)
    yb, Fb = O.ttt_mlp_minibatch(q[split:], k[split:], v[split:], eta[split:], *Fa, chunk)
    np.testing.assert_allclose(np.concatenate([ya, yb]), y, rtol=1e-12, atol=1e-12)
    for a, b in zip(Fb, F):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_outputs_are_causal():
    """Changing token t+1.. leaves y_0..y_t unchanged (the chunk-start
    weights do not see later tokens of the chunk)."""
    rng = np.random.default_rng(7)
    P = params(rng, 3, 5, 4)
    q, k, v, eta = tokens(rng, 10, 3, 4)
    y, _ = O.ttt_mlp_minibatch(q, k, v, eta, *P, 4)
    k2, v2 = k.copy(), v.copy()
    k2[6:] += 1.0
    v2[6:] -= 1.0
    y2, _ = O.ttt_mlp_minibatch(q, k2, v2, eta, *P, 4)
    np.testing.assert_array_equal(y[:6], y2[:6])
    assert np.abs(y[6:] - y2[6:]).max() > 1e-6
