"""The synthetic inputs follow the stated recipe, and the binding's
descriptors carry what the C ABI expects (CPU only)."""
import numpy as np
import pytest
import torch

from linear_attention_ttt_b200 import ops, synth


def test_workloads_are_deterministic_and_replicas_differ():
    a, b = synth.config(2, T=64), synth.config(2, T=64)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.eta, b.eta)
    c = synth.config(2, T=64, replica=1)
    assert not np.array_equal(a.q, c.q)


def test_bf16_workloads_hold_bf16_values():
    w = synth.config(3, T=64)
    for x in (w.q, w.k, w.v):
        assert np.array_equal(synth.round_to_bf16(x), x)


@pytest.mark.parametrize("index", [1, 3])
def test_mse_workloads_normalise_q_and_k(index):
    w = synth.config(index, T=64)
    tol = 1e-6 if w.dtype == synth.F32 else 2 ** -7
    for x in (w.q, w.k):
        assert np.abs(np.linalg.norm(x.astype(np.float64), axis=-1) - 1.0).max() < tol


def test_learning_rate_distributions():
    e1 = synth.config(1, T=64).eta
    assert np.all(e1 == np.float32(0.1))
    e2 = synth.config(2, T=256).eta
    assert e2.min() > 0 and e2.max() < 0.1          # 0.1 * sigmoid(.)
    e3 = synth.config(3, T=256).eta
    assert e3.min() > 0 and np.isfinite(e3).all()   # 0.05 * softplus(.)


def test_linear_attention_workload_starts_from_zero_state():
    w = synth.config(2, T=64)
    assert np.all(w.W0 == 0)
    assert w.dk == w.dv == 128 and w.chunk == 64 and w.loss == synth.LOSS_NEG_DOT


def test_descriptors_of_permuted_and_empty_tensors():
    x = torch.zeros(2, 5, 3, 8).permute(0, 2, 1, 3)      # [B,H,T,d] view of [B,T,H,d]
    d = ops.describe(x)
    assert d.ndim == 4 and d.dtype == ops.TTT_F32
    assert [d.shape[i] for i in range(4)] == [2, 3, 5, 8]
    assert [d.stride[i] for i in range(4)] == list(x.stride())
    assert d.data == x.data_ptr()
    e = ops.describe(torch.zeros(2, 3, 0, 8, dtype=torch.bfloat16))
    assert e.data in (0, None) and e.dtype == ops.TTT_BF16 and e.shape[2] == 0
    assert ops.describe(None) is None
    with pytest.raises(TypeError):
        ops.describe(torch.zeros(2, dtype=torch.float16))
