"""GPU parity of lact_swiglu_bwd (C ABI) against the fp64 autograd oracle
(oracle.lact_backward.lact_swiglu_bwd, pinned by finite differences of the
numpy LaCT forward)."""
import numpy as np
import pytest
import torch

from oracle import lact_backward as LB
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, dev

pytestmark = pytest.mark.gpu


def compare(w, what, seed=0, with_final=True, per_seq=False):
    rng = np.random.default_rng(seed)
    rnd = synth.round_to_bf16 if w.dtype == synth.BF16 else synth.round_to_f32
    dy = rnd(rng.standard_normal(w.v.shape))
    Ws = [w.W1, w.W2, w.W3]
    if per_seq:
        Ws = [synth.round_to_f32(np.broadcast_to(W, (w.B,) + W.shape) *
                                 (1 + 0.1 * rng.standard_normal((w.B,) + W.shape))) for W in Ws]
    dWf = None
    if with_final:
        dWf = [synth.round_to_f32(rng.standard_normal((w.B, w.H) + W.shape[-2:])) for W in Ws]
    t = [dev(x, w.dtype) for x in (w.q, w.k, w.v)]
    got = ops.lact_swiglu_bwd(*t, dev(w.eta, synth.F32), *[dev(W, synth.F32) for W in Ws],
                              w.chunk, w.update_rule, w.causal, dev(dy, w.dtype),
                              tuple(dev(x, synth.F32) for x in dWf) if dWf else (None,) * 3)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    got = [x.float().cpu().numpy().astype(np.float64) for x in got]
    want = LB.lact_swiglu_bwd(w.q, w.k, w.v, w.eta, *Ws, w.chunk, w.update_rule, w.causal, dy, dWf)
    for g, o, n in zip(got, want, ("dq", "dk", "dv", "deta", "dW1", "dW2", "dW3")):
        if n == "deta":
            g, o = g.reshape(-1, w.T), o.reshape(-1, w.T)
        check(g, o, w.dtype, f"{what} {n}")


@pytest.mark.parametrize("rule", [synth.UPDATE_GD, synth.UPDATE_MUON])
@pytest.mark.parametrize("causal", [1, 0])
def test_bf16_small(rule, causal):
    w = synth.make_lact(1, 2, 256, 64, 128, 64, rule, seed=60 + rule + 2 * causal, causal=causal,
                        eta_scale=0.05)
    compare(w, f"rule{rule} causal{causal}", seed=rule + causal)


def test_f32_gd_ragged_per_sequence_weights():
    w = synth.make_lact(2, 1, 150, 64, 128, 64, synth.UPDATE_GD, seed=64, dtype=synth.F32,
                        eta_scale=0.05)
    compare(w, "f32 gd ragged per-seq", seed=4, per_seq=True)


def test_bf16_muon_d128_hidden512_without_final_gradient():
    """The Muon workload's head and hidden sizes (128, 512), 3 chunks."""
    w = synth.make_lact(1, 1, 384, 128, 512, 128, synth.UPDATE_MUON, seed=65)
    compare(w, "muon d128 dh512", seed=5, with_final=False)
