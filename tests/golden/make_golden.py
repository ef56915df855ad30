"""Writes tests/golden/oracle_small_cases.json: oracle outputs on a few tiny
seeded cases, kept as regression values so that any later change to the
oracle's arithmetic shows up as a failing pin. Calls only oracle/ and the
seeded input generator. Run: python -m tests.golden.make_golden
"""
import json
import os

import numpy as np

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import synth

CASES = ["mse_f32_T20_b8", "negdot_f32_T20_b8", "lact_gd_T10_b4", "lact_muon_T10_b4"]


def compute(name):
    if name.startswith("mse") or name.startswith("negdot"):
        loss = O.LOSS_MSE if name.startswith("mse") else O.LOSS_NEG_DOT
        w = synth.make_ttt_linear(1, 1, 20, 4, 3, 8, synth.F32, loss, seed=42,
                                  eta_kind="softplus", eta_scale=0.2, w0_std=0.5)
        y, W = O.ttt_linear_minibatch(w.q, w.k, w.v, w.eta, w.W0, 8, loss)
        return {"y": y.ravel().tolist(), "W_final": W.ravel().tolist()}
    rule = O.UPDATE_GD if "gd" in name else O.UPDATE_MUON
    w = synth.make_lact(1, 1, 10, 3, 5, 4, rule, seed=43, dtype=synth.F32, eta_scale=0.3)
    y, F1, F2, F3 = O.lact_swiglu(w.q, w.k, w.v, w.eta, w.W1, w.W2, w.W3, 4, rule, 1)
    return {"y": y.ravel().tolist(), "W1_final": F1.ravel().tolist(),
            "W2_final": F2.ravel().tolist(), "W3_final": F3.ravel().tolist()}


def main():
    out = {"_source": "oracle outputs (fp64) on seeded tiny cases; regression values written by tests/golden/make_golden.py"}
    for name in CASES:
        out[name] = compute(name)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_cases.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
        f.write("\n")


if __name__ == "__main__":
    main()
