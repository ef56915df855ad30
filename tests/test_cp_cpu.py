"""Context-parallel LaCT on CPU ranks (gloo, world size 2): the token split of
linear_attention_ttt_b200.cp and a per-chunk all-reduce of the gradients give
the single-device layer ("Test-Time Training Done Right" review, section 8:
each device computes the gradient of its share of a chunk, the shares are
summed). The arithmetic per rank is the oracle's; what is checked is the
decomposition and the shard layout."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import cp, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def cp_scan(q, k, v, eta, W1, W2, W3, chunk_local, rule, causal):
    """One rank's share of the layer: per chunk, the oracle's gradient of the
    local tokens, summed over the ranks, then the replicated update."""
    w = [np.array(W, dtype=np.float64) for W in (W1, W2, W3)]
    rho = [O.row_norms(x) for x in w]
    y = np.zeros(v.shape)
    for s in range(0, q.shape[0], chunk_local):
        e = s + chunk_local
        if causal:
            y[s:e] = O.swiglu(*w, q[s:e])
        g = O.lact_grads(*w, k[s:e], v[s:e], eta[s:e])
        flat = torch.from_numpy(np.concatenate([x.ravel() for x in g]))
        dist.all_reduce(flat)
        parts, off = [], 0
        for x in g:
            parts.append(flat[off:off + x.size].numpy().reshape(x.shape))
            off += x.size
        if rule == O.UPDATE_MUON:
            parts = [O.newton_schulz5(x) for x in parts]
        w = [O.renorm_rows(x - gx, r) for x, gx, r in zip(w, parts, rho)]
        if not causal:
            y[s:e] = O.swiglu(*w, q[s:e])
    return y, w


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for rule, causal in ((O.UPDATE_GD, 1), (O.UPDATE_MUON, 1), (O.UPDATE_GD, 0)):
            w = synth.make_lact(1, 1, 48, 4, 6, 12, rule, seed=30 + rule + 2 * causal,
                                dtype=synth.F32, eta_scale=0.1)
            sh = lambda x: cp.shard(torch.from_numpy(np.asarray(x, np.float64)), rank, world,
                                    w.chunk).numpy()
            q, k, v = (sh(x)[0, 0] for x in (w.q, w.k, w.v))
            eta = sh(w.eta[..., None])[0, 0, :, 0]
            y, fin = cp_scan(q, k, v, eta, w.W1[0], w.W2[0], w.W3[0], w.chunk // world, rule,
                             causal)
            res[(rule, causal)] = (y, fin)
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_two_ranks_equal_the_single_device_layer():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rule, causal in ((O.UPDATE_GD, 1), (O.UPDATE_MUON, 1), (O.UPDATE_GD, 0)):
        w = synth.make_lact(1, 1, 48, 4, 6, 12, rule, seed=30 + rule + 2 * causal,
                            dtype=synth.F32, eta_scale=0.1)
        yo, F1, F2, F3 = O.lact_swiglu(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, w.chunk, rule,
                                       causal)
        parts = [torch.from_numpy(out[r][(rule, causal)][0][None, None]) for r in range(world)]
        y = cp.unshard(parts, w.chunk).numpy()[0, 0]
        np.testing.assert_allclose(y, yo[0, 0], rtol=1e-10, atol=1e-12)
        for r in range(world):   # the weights are the same on every rank
            for a, b in zip(out[r][(rule, causal)][1], (F1[0, 0], F2[0, 0], F3[0, 0])):
                np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_shard_and_unshard_are_inverse():
    x = torch.arange(2 * 3 * 24 * 5).reshape(2, 3, 24, 5)
    for world, chunk in ((2, 8), (4, 8), (3, 12), (1, 6)):
        parts = [cp.shard(x, r, world, chunk) for r in range(world)]
        assert all(p.shape == (2, 3, 24 // world, 5) for p in parts)
        assert torch.equal(cp.unshard(parts, chunk), x)
    # rank 1 of 2 with chunk 8 holds tokens 4-7, 12-15, 20-23
    assert cp.shard(x, 1, 2, 8)[0, 0, :, 0].tolist() == [5 * t for t in (4, 5, 6, 7, 12, 13, 14, 15, 20, 21, 22, 23)]
