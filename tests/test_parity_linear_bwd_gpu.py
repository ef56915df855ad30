"""GPU parity of ttt_linear_bwd (C ABI) against the fp64 oracle's reverse
chunk scan (oracle.ttt_oracle.ttt_linear_minibatch_bwd, itself pinned by
finite differences of the forward definition)."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, dev, upload_linear

pytestmark = pytest.mark.gpu


def run(w, dy, dWf):
    t = upload_linear(w)
    dyd = dev(dy, w.dtype)
    dWfd = dev(dWf, synth.F32) if dWf is not None else None
    outs = ops.ttt_linear_bwd(t["q"], t["k"], t["v"], t["eta"], t["W0"], w.chunk, w.loss, dyd,
                              dWfd)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return [x.float().cpu().numpy().astype(np.float64) for x in outs]


def compare(w, what, seed=0, with_dwf=True):
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal(w.v.shape)
    dy = synth.round_to_bf16(dy) if w.dtype == synth.BF16 else synth.round_to_f32(dy)
    dWf = synth.round_to_f32(rng.standard_normal((w.B, w.H, w.dk, w.dv))) if with_dwf else None
    got = run(w, dy, dWf)
    want = O.ttt_linear_minibatch_bwd(w.q, w.k, w.v, w.eta, w.W0, w.chunk, w.loss, dy, dWf)
    for g, o, n in zip(got, want, ("dq", "dk", "dv", "deta", "dW0")):
        if n != "dW0" and w.T == 0:   # no tokens: only the weight gradient exists
            assert g.size == 0
            continue
        if n == "deta":   # one value per token: compare as one row per (batch, head)
            g, o = g.reshape(-1, w.T), o.reshape(-1, w.T)
        check(g, o, w.dtype, f"{what} {n}")


@pytest.mark.parametrize("loss", [synth.LOSS_MSE, synth.LOSS_NEG_DOT])
@pytest.mark.parametrize("T,chunk", [(40, 16), (37, 5), (16, 1), (50, 64)])
def test_f32_ragged_chunks(loss, T, chunk):
    w = synth.make_ttt_linear(2, 2, T, 32, 48, chunk, synth.F32, loss, seed=T + chunk,
                              eta_kind="softplus", eta_scale=0.1, w0_std=0.1)
    compare(w, f"f32 loss{loss} T{T} b{chunk}", seed=T)


@pytest.mark.parametrize("loss", [synth.LOSS_MSE, synth.LOSS_NEG_DOT])
def test_f32_per_sequence_w0_and_no_final_gradient(loss):
    w = synth.make_ttt_linear(2, 3, 33, 16, 16, 8, synth.F32, loss, seed=9, eta_kind="sigmoid",
                              eta_scale=0.2, w0_std=0.1, w0_batched=True)
    compare(w, f"f32 batched W0 loss{loss}", seed=3, with_dwf=False)


def test_bf16_mse_workload_shape():
    """Small-chunk TTT-Linear MSE (d 64, chunk 16, bf16 tokens) on a shortened
    sequence: two sequences of the workload's distribution."""
    w = synth.config(3, B=1, H=2, T=512)
    compare(w, "bf16 mse config3 T512", seed=5)


def test_bf16_inner_product_workload_shape():
    """Inner-product layer (d 128, chunk 64, bf16 tokens), shortened."""
    w = synth.config(2, B=1, H=2, T=320)
    compare(w, "bf16 la config2 T320", seed=6)


def test_f32_workload_1():
    """The fp32 MSE workload (B1 H2 T256 d64 chunk 16) at full size."""
    compare(synth.config(1), "config1", seed=1)


def test_empty_sequence():
    w = synth.make_ttt_linear(1, 2, 0, 16, 16, 4, synth.F32, synth.LOSS_MSE, seed=2)
    compare(w, "T0", seed=2)
