"""GPU parity of window_attention_fwd and lact_swiglu_window_fwd (C ABI)
against the fp64 oracle (oracle.ttt_oracle.sliding_window_attention, pinned
by torch's causal attention, a banded brute force and window 1)."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, dev, upload_lact

pytestmark = pytest.mark.gpu


def tokens(B, H, T, d, seed):
    w = synth.make_lact(B, H, T, d, 2 * d, 64, synth.UPDATE_GD, seed)
    return w


def oracle_attn(w, window):
    y = np.zeros(w.v.shape)
    for b in range(w.B):
        for h in range(w.H):
            y[b, h] = O.sliding_window_attention(w.q[b, h], w.k[b, h], w.v[b, h], window)
    return y


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("T,window", [(200, 64), (130, 1), (257, 100), (96, 4096), (64, 63)])
def test_window_attention_matches_oracle(d, T, window):
    w = tokens(1, 2, T, d, seed=T + window + d)
    t = [dev(x, w.dtype) for x in (w.q, w.k, w.v)]
    y = ops.window_attention_fwd(*t, window)
    torch.cuda.synchronize()
    check(y.float().cpu().numpy(), oracle_attn(w, window), w.dtype, f"d{d} T{T} w{window}")


def test_accumulate_adds_into_out():
    w = tokens(2, 1, 150, 128, seed=5)
    t = [dev(x, w.dtype) for x in (w.q, w.k, w.v)]
    base = torch.randn_like(t[2]) * 0.1
    out = base.clone()
    ops.window_attention_fwd(*t, 48, out=out, accumulate=True)
    torch.cuda.synchronize()
    want = base.float().cpu().numpy() + oracle_attn(w, 48)
    check(out.float().cpu().numpy(), want, w.dtype, "accumulate")


def test_window_4096_over_a_long_sequence():
    """The pages' language-model window (4K tokens) over 8K tokens, d 128."""
    w = tokens(1, 1, 8192, 128, seed=7)
    t = [dev(x, w.dtype) for x in (w.q, w.k, w.v)]
    y = ops.window_attention_fwd(*t, 4096).float().cpu().numpy()
    torch.cuda.synchronize()
    rows = np.r_[0:64, 4000:4200, 8100:8192]
    ref = O.sliding_window_attention(w.q[0, 0], w.k[0, 0], w.v[0, 0], 4096)[rows]
    check(y[0, 0, rows], ref, w.dtype, "w4096 sampled rows")


@pytest.mark.parametrize("rule", [synth.UPDATE_GD, synth.UPDATE_MUON])
def test_lact_with_window_attention(rule):
    w = synth.make_lact(1, 2, 640, 128, 512, 128, rule, seed=11 + rule, eta_scale=0.02)
    t = upload_lact(w)
    y = ops.lact_swiglu_window_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"],
                                   w.chunk, rule, 256)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    ref = np.stack([np.stack([O.lact_with_window_attention(w.q[b, h], w.k[b, h], w.v[b, h],
                                                           w.eta[b, h], w.W1[h], w.W2[h], w.W3[h],
                                                           w.chunk, rule, 256)
                              for h in range(w.H)]) for b in range(w.B)])
    check(y.float().cpu().numpy(), ref, w.dtype, f"lact+window rule{rule}")
