"""GPU parity of lact_swiglu_fwd (C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, run_lact, upload_lact

pytestmark = pytest.mark.gpu


def oracle(w):
    return O.lact_swiglu(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, w.chunk, w.update_rule, w.causal)


def compare(w, what=""):
    y, F1, F2, F3 = run_lact(w)
    yo, O1, O2, O3 = oracle(w)
    r = [check(y, yo, w.dtype, what + " y")]
    for g, o, n in ((F1, O1, "W1"), (F2, O2, "W2"), (F3, O3, "W3")):
        r.append(check(g, o, w.dtype, f"{what} {n}_final"))
    return r


@pytest.mark.parametrize("d,dh", [(64, 128), (128, 256), (256, 512)])
def test_gd_causal_small(d, dh):
    w = synth.make_lact(1, 2, 512, d, dh, 128, synth.UPDATE_GD, seed=d + dh, eta_scale=0.02)
    compare(w, f"gd d{d}")


@pytest.mark.parametrize("T,chunk", [(300, 128), (200, 64), (64, 256), (1, 16)])
def test_gd_ragged_chunks(T, chunk):
    w = synth.make_lact(2, 1, T, 128, 256, chunk, synth.UPDATE_GD, seed=T, eta_scale=0.02)
    compare(w, f"gd T{T} b{chunk}")


def test_gd_non_causal():
    w = synth.make_lact(1, 2, 384, 128, 256, 128, synth.UPDATE_GD, seed=3, causal=0,
                        eta_scale=0.02)
    compare(w, "gd non-causal")


def test_muon_small():
    """d = 128, hidden 512: the shared-memory-resident Newton-Schulz path."""
    w = synth.make_lact(1, 2, 1024, 128, 512, 256, synth.UPDATE_MUON, seed=5)
    compare(w, "muon")


@pytest.mark.parametrize("d,dh", [(64, 128), (256, 512), (128, 256)])
def test_muon_other_shapes(d, dh):
    """Gradient shapes outside 128 x 512 take the general cluster Newton-Schulz."""
    w = synth.make_lact(1, 2, 512, d, dh, 256, synth.UPDATE_MUON, seed=d + dh + 1)
    compare(w, f"muon d{d} dh{dh}")


def test_gd_full_size_workload():
    """LaCT GD: batch 2, 4 heads, T=32768, d=256, hidden 512, chunk 2048."""
    compare(synth.config(4), "config4")


def test_muon_full_size_workload():
    """LaCT Muon: batch 1, 8 heads, T=131072, d=128, hidden 512, chunk 4096."""
    compare(synth.config(5), "config5")


def test_causal_outputs_ignore_later_chunks():
    """Apply-then-update: perturbing chunk c's keys, values and learning rates
    leaves every output up to and including chunk c bit-identical."""
    w = synth.make_lact(1, 2, 512, 128, 256, 128, synth.UPDATE_GD, seed=9, eta_scale=0.05)
    t = upload_lact(w)
    y0 = ops.lact_swiglu_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"], 128)
    c = 2
    for n in ("k", "v", "eta"):
        t[n][:, :, c * 128:(c + 1) * 128] *= 1.5
    y1 = ops.lact_swiglu_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"], 128)
    torch.cuda.synchronize()
    assert torch.equal(y0[:, :, :(c + 1) * 128], y1[:, :, :(c + 1) * 128])
    assert not torch.equal(y0[:, :, (c + 1) * 128:], y1[:, :, (c + 1) * 128:])


def test_zero_learning_rate_keeps_weights():
    w = synth.make_lact(1, 2, 256, 128, 256, 64, synth.UPDATE_GD, seed=2)
    w.eta[:] = 0
    y, F1, F2, F3 = run_lact(w)
    assert np.array_equal(F1, np.broadcast_to(w.W1, F1.shape))
    assert np.array_equal(F2, np.broadcast_to(w.W2, F2.shape))
    ref = np.stack([np.stack([O.swiglu(w.W1[h], w.W2[h], w.W3[h], w.q[b, h]) for h in range(w.H)])
                    for b in range(w.B)])
    check(y, ref, w.dtype, "eta=0 y")


def test_empty_sequence_copies_weights():
    w = synth.make_lact(1, 2, 0, 128, 256, 64, synth.UPDATE_GD, seed=2)
    y, F1, F2, F3 = run_lact(w)
    assert np.array_equal(F3, np.broadcast_to(w.W3, F3.shape))
