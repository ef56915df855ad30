"""Pins of the window-attention oracle (the scope table's "next" row f4),
CPU only."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O


def data(T, d, dv, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((T, d)), rng.standard_normal((T, d)), rng.standard_normal((T, dv))


def test_a_window_covering_the_sequence_is_causal_attention():
    """Against torch's scaled-dot-product attention with a causal mask."""
    q, k, v = data(12, 8, 5, 1)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], is_causal=True)[0]
    np.testing.assert_allclose(O.sliding_window_attention(q, k, v, 12), want.numpy(),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.sliding_window_attention(q, k, v, 100), want.numpy(),
                               rtol=1e-12, atol=1e-12)


def test_window_one_returns_the_token_value():
    q, k, v = data(7, 4, 3, 2)
    np.testing.assert_allclose(O.sliding_window_attention(q, k, v, 1), v, rtol=0, atol=0)


@pytest.mark.parametrize("window", [2, 3, 5])
def test_window_matches_a_banded_mask(window):
    """Brute force with an explicit band mask: i in (t - window, t]."""
    q, k, v = data(10, 4, 3, window)
    s = q @ k.T / 2.0
    t, i = np.indices(s.shape)
    s = np.where((i <= t) & (i > t - window), s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    want = (p / p.sum(axis=1, keepdims=True)) @ v
    np.testing.assert_allclose(O.sliding_window_attention(q, k, v, window), want,
                               rtol=1e-12, atol=1e-12)


def test_combined_layer_is_the_sum_of_both_branches():
    rng = np.random.default_rng(3)
    T, d, dh = 8, 4, 8
    q, k, v = data(T, d, d, 4)
    eta = 0.1 * rng.random(T)
    W1 = rng.standard_normal((dh, d)) / 2
    W2 = rng.standard_normal((d, dh)) / 3
    W3 = rng.standard_normal((dh, d)) / 2
    y = O.lact_with_window_attention(q, k, v, eta, W1, W2, W3, 4, O.UPDATE_GD, 3)
    ya, *_ = O.lact_swiglu(q[None, None], k[None, None], v[None, None], eta[None, None], W1[None],
                           W2[None], W3[None], 4, O.UPDATE_GD, 1)
    np.testing.assert_allclose(y - O.sliding_window_attention(q, k, v, 3), ya[0, 0], rtol=1e-12,
                               atol=1e-12)
