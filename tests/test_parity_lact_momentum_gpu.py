"""GPU parity of lact_swiglu_fwd_momentum (C ABI) against the fp64 oracle's
momentum scan (heavy-ball momentum on the chunk gradients, the reading the
"Test-Time Training Done Right" review's section 3.3 leaves open)."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, dev, upload_lact

pytestmark = pytest.mark.gpu


def run(w, beta, M0=None):
    t = upload_lact(w)
    m0 = tuple(dev(m, synth.F32) for m in M0) if M0 is not None else (None, None, None)
    out, F, M = ops.lact_swiglu_fwd_momentum(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                             t["W3"], w.chunk, beta, w.causal, M0=m0, finals=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    f = lambda x: x.float().cpu().numpy().astype(np.float64)
    return f(out), [f(x) for x in F], [f(x) for x in M]


def compare(w, beta, what, M0=None):
    y, F, M = run(w, beta, M0)
    yo, O1, O2, O3, Mo = O.lact_swiglu_momentum(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, w.chunk,
                                                beta, w.causal, M0=M0)
    check(y, yo, w.dtype, what + " y")
    for g, o, n in zip(F, (O1, O2, O3), ("W1", "W2", "W3")):
        check(g, o, w.dtype, f"{what} {n}_final")
    for g, o, n in zip(M, Mo, ("M1", "M2", "M3")):
        check(g, o, w.dtype, f"{what} {n}_final")


@pytest.mark.parametrize("d,dh,beta", [(128, 256, 0.9), (64, 128, 0.5), (256, 512, 0.9)])
def test_momentum_matches_oracle(d, dh, beta):
    w = synth.make_lact(1, 2, 640, d, dh, 128, synth.UPDATE_GD, seed=40 + d, eta_scale=0.02)
    compare(w, beta, f"momentum d{d} beta{beta}")


def test_momentum_ragged_non_causal_and_initial_momentum():
    w = synth.make_lact(2, 1, 300, 128, 256, 128, synth.UPDATE_GD, seed=44, causal=0,
                        eta_scale=0.02)
    rng = np.random.default_rng(4)
    M0 = tuple(synth.round_to_f32(1e-3 * rng.standard_normal(W.shape)) for W in (w.W1, w.W2, w.W3))
    compare(w, 0.8, "momentum non-causal M0", M0=M0)


def test_beta_zero_is_gd_bit_for_bit():
    """beta = 0: the step beta * M + G is G exactly, so the momentum path
    runs the GD computation and must give the same bits."""
    w = synth.make_lact(1, 2, 512, 128, 256, 128, synth.UPDATE_GD, seed=45, eta_scale=0.02)
    t = upload_lact(w)
    y0, *F0 = ops.lact_swiglu_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"],
                                  w.chunk, finals=True)
    y1, F1, _ = ops.lact_swiglu_fwd_momentum(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                             t["W3"], w.chunk, 0.0, finals=True)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    for a, b in zip(F0, F1):
        assert torch.equal(a, b)


def test_momentum_full_size_gd_workload_shape():
    """The LaCT GD workload's shape (d 256, hidden 512, chunk 2048) on a
    shortened sequence of 4 chunks, beta 0.9."""
    w = synth.config(4, T=8192)
    compare(w, 0.9, "momentum config4 T8192")
