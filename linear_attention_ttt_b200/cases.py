"""Run one entry point of the library on a named synthetic case, a few times,
for profilers (ncu captures of a single kernel on a small case).

    python -m linear_attention_ttt_b200.cases <case> [--reps N]

Cases (synthetic inputs with the workloads' distributions, shortened):
  window       window attention, B1 H8 T16384 d128, window 4096
  lact_window  the LaCT Muon layer plus window attention, B1 H8 T16384 d128 dh512 b4096
  ttt_mlp      TTT-MLP, B4 H16 T2048 d64 dh256 chunk 16, bf16
  linear_bwd   TTT-Linear MSE backward, B8 H16 T2048 d64 chunk 16, bf16
  lact_bwd     LaCT GD backward, B1 H2 T2048 d128 dh512 chunk 1024, bf16
  momentum     LaCT with momentum (beta 0.9), B2 H4 T8192 d256 dh512 chunk 2048
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from . import ops, synth


def _dev(x, dtype):
    a = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return a.to(torch.bfloat16) if dtype == synth.BF16 else a


def _lact_tensors(w):
    return {n: _dev(getattr(w, n), w.dtype if n in ("q", "k", "v") else synth.F32)
            for n in ("q", "k", "v", "eta", "W1", "W2", "W3")}


def make_case(name):
    """Returns a callable that runs the case once (inputs resident on the GPU)."""
    if name in ("window", "lact_window"):
        w = synth.config(5, T=16384)
        t = _lact_tensors(w)
        out = torch.empty_like(t["v"])
        if name == "window":
            return lambda: ops.window_attention_fwd(t["q"], t["k"], t["v"], 4096, out=out)
        return lambda: ops.lact_swiglu_window_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"],
                                                  t["W2"], t["W3"], w.chunk, w.update_rule,
                                                  4096, out=out)
    if name == "ttt_mlp":
        w = synth.config(3, B=4, T=2048)
        rng = np.random.default_rng(7)
        P = [rng.standard_normal((w.H, 256, 64)) / 8, np.zeros((w.H, 256)),
             rng.standard_normal((w.H, 64, 256)) / 16, np.zeros((w.H, 64))]
        t = [_dev(getattr(w, n), w.dtype) for n in ("q", "k", "v")] + [_dev(w.eta, synth.F32)]
        Pd = [_dev(p, synth.F32) for p in P]
        return lambda: ops.ttt_mlp_fwd(*t, *Pd, 16)
    if name == "linear_bwd":
        w = synth.config(3, T=2048)
        t = [_dev(getattr(w, n), w.dtype if n in ("q", "k", "v") else synth.F32)
             for n in ("q", "k", "v", "eta", "W0")]
        dy = torch.randn_like(t[2])
        return lambda: ops.ttt_linear_bwd(*t, w.chunk, w.loss, dy)
    if name == "lact_bwd":
        w = synth.make_lact(1, 2, 2048, 128, 512, 1024, synth.UPDATE_GD, seed=1090)
        t = _lact_tensors(w)
        dy = torch.randn_like(t["v"])
        return lambda: ops.lact_swiglu_bwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                           t["W3"], w.chunk, 0, 1, dy)
    if name == "momentum":
        w = synth.config(4, T=8192)
        t = _lact_tensors(w)
        out = torch.empty_like(t["v"])
        return lambda: ops.lact_swiglu_fwd_momentum(t["q"], t["k"], t["v"], t["eta"], t["W1"],
                                                    t["W2"], t["W3"], w.chunk, 0.9, out=out)
    raise ValueError(f"unknown case {name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    ops.load()
    fn = make_case(args.case)
    for _ in range(args.reps):
        fn()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    print(f"{args.case}: {args.reps} runs ok")


if __name__ == "__main__":
    main()
