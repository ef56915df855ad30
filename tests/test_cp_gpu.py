"""GPU checks of lact_swiglu_fwd_cp (C ABI) on the one GPU a run has: with no
exchange it is lact_swiglu_fwd bit for bit; with a one-rank NCCL group it is
the same; and its per-chunk gradient hook really feeds the update: a chunk
made of two identical halves, run as one shard with a hook that doubles the
gradient (the sum two ranks holding those halves would form), matches the
oracle on the whole duplicated sequence."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import cp, ops, synth
from tests.gpu_util import check, dev, upload_lact

pytestmark = pytest.mark.gpu


def test_no_exchange_is_the_plain_layer():
    w = synth.make_lact(1, 2, 512, 128, 256, 128, synth.UPDATE_MUON, seed=50, eta_scale=0.02)
    t = upload_lact(w)
    args = (t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"], w.chunk, w.update_rule)
    y0, *F0 = ops.lact_swiglu_fwd(*args, finals=True)
    y1, *F1 = cp.lact_swiglu_fwd_cp(*args, None, finals=True)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    for a, b in zip(F0, F1):
        assert torch.equal(a, b)


def test_one_rank_nccl_group():
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.make_lact(1, 2, 512, 128, 256, 128, synth.UPDATE_GD, seed=51, eta_scale=0.02)
        t = upload_lact(w)
        args = (t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"], w.chunk, 0)
        y0 = ops.lact_swiglu_fwd(*args)
        red = cp.dist_reducer()
        y1 = cp.lact_swiglu_fwd_cp(*args, red)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("rule", [synth.UPDATE_GD, synth.UPDATE_MUON])
def test_gradient_hook_feeds_the_update(rule):
    half = synth.make_lact(1, 2, 1024, 128, 512, 128, rule, seed=52 + rule, eta_scale=0.01)
    # the full sequence: every chunk of 256 tokens is a 128-token block twice
    def dup(x):
        B, H, T = x.shape[:3]
        v = x.reshape(B, H, T // 128, 1, 128, *x.shape[3:])
        return np.concatenate([v, v], axis=3).reshape(B, H, 2 * T, *x.shape[3:])
    q, k, v, eta = (dup(x) for x in (half.q, half.k, half.v, half.eta))
    yo, O1, O2, O3 = O.lact_swiglu(q, k, v, eta, half.W1, half.W2, half.W3, 256, rule, 1)
    t = upload_lact(half)
    red = cp.make_reducer(lambda g: g.mul_(2.0))
    y, F1, F2, F3 = cp.lact_swiglu_fwd_cp(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                          t["W3"], 128, rule, red, finals=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    yo_half = yo.reshape(1, 2, -1, 2, 128, yo.shape[-1])[:, :, :, 0].reshape(y.shape)
    f = lambda x: x.float().cpu().numpy()
    check(f(y), yo_half, half.dtype, f"cp hook rule{rule} y")
    for g, o, n in ((F1, O1, "W1"), (F2, O2, "W2"), (F3, O3, "W3")):
        check(f(g), o, half.dtype, f"cp hook rule{rule} {n}")
