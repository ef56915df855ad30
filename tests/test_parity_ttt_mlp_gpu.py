"""GPU parity of ttt_mlp_fwd (C ABI) against the fp64 oracle's TTT-MLP
mini-batch rule (oracle.ttt_oracle.ttt_mlp_minibatch), sequence by sequence."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, dev

pytestmark = pytest.mark.gpu


def case(B, H, T, dk, dv, dh, chunk, dtype, seed, per_seq=False):
    """Tokens of the TTT-Linear recipe (q, k L2-normalised) and MLP parameters
    W ~ N(0, 1/fan_in), small biases."""
    w = synth.make_ttt_linear(B, H, T, dk, dv, chunk, dtype, synth.LOSS_MSE, seed,
                              eta_kind="softplus", eta_scale=0.05, w0_std=0.0)
    rng = np.random.default_rng(seed + 1)
    lead = (B, H) if per_seq else (H,)
    P = [rng.standard_normal(lead + (dh, dk)) / np.sqrt(dk), 0.1 * rng.standard_normal(lead + (dh,)),
         rng.standard_normal(lead + (dv, dh)) / np.sqrt(dh), 0.1 * rng.standard_normal(lead + (dv,))]
    return w, [synth.round_to_f32(p) for p in P]


def compare(w, P, what):
    t = [dev(x, w.dtype) for x in (w.q, w.k, w.v)]
    out, *F = ops.ttt_mlp_fwd(*t, dev(w.eta, synth.F32), *[dev(p, synth.F32) for p in P],
                              w.chunk, finals=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    f = lambda x: x.float().cpu().numpy().astype(np.float64)
    y, F = f(out), [f(x) for x in F]
    per_seq = P[0].ndim == 4
    yo = np.zeros_like(y)
    Fo = [np.zeros_like(x) for x in F]
    for b in range(w.B):
        for h in range(w.H):
            ps = [p[b, h] if per_seq else p[h] for p in P]
            yo[b, h], fo = O.ttt_mlp_minibatch(w.q[b, h], w.k[b, h], w.v[b, h], w.eta[b, h], *ps,
                                               w.chunk)
            for i in range(4):
                Fo[i][b, h] = fo[i]
    check(y, yo, w.dtype, what + " y")
    for g, o, n in zip(F, Fo, ("W1", "b1", "W2", "b2")):
        if g.ndim == 3:   # biases: one row per (batch, head)
            g, o = g[..., None, :], o[..., None, :]
        check(g, o, w.dtype, f"{what} {n}_final")


@pytest.mark.parametrize("T,chunk", [(64, 16), (53, 16), (40, 7), (16, 1), (37, 64)])
def test_f32_chunks(T, chunk):
    w, P = case(2, 2, T, 32, 32, 128, chunk, synth.F32, seed=T + chunk)
    compare(w, P, f"f32 T{T} b{chunk}")


def test_bf16_head64_hidden256():
    """Head dim 64 and hidden 4 x 64 (the usual TTT-MLP width), chunk 16."""
    w, P = case(1, 2, 256, 64, 64, 256, 16, synth.BF16, seed=11)
    compare(w, P, "bf16 d64 dh256")


def test_per_sequence_parameters_and_uneven_sizes():
    w, P = case(2, 1, 50, 48, 16, 96, 16, synth.F32, seed=12, per_seq=True)
    compare(w, P, "f32 per-seq")


def test_empty_sequence_copies_parameters():
    w, P = case(1, 2, 0, 32, 32, 64, 16, synth.F32, seed=13)
    compare(w, P, "T0")


@pytest.mark.parametrize("chunk", [16, 32])
def test_parameters_beyond_shared_memory(chunk):
    """dk = dv = 128, dh = 512: the parameters (527 KB) do not fit in shared
    memory, so both copies stay in the workspace."""
    w, P = case(1, 1, 50, 128, 128, 512, chunk, synth.F32, seed=14 + chunk)
    compare(w, P, f"f32 d128 dh512 b{chunk}")
