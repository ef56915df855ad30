"""Helpers shared by the GPU parity tests: upload seeded workloads, run the
CUDA path through the C ABI, and the error metrics the tolerances apply to.

Metrics (applied to y and to the final weights):
  max_row_rel: max over rows r of max_j |g_rj - o_rj| / max_j |o_rj|, a row
               being one token's head output or one row of a weight matrix;
  rel_frob:    ||g - o||_F / ||o||_F over the whole tensor.
Tolerances: fp32 tokens max_row_rel <= 1e-4; bf16 tokens with fp32 state
max_row_rel <= 2e-2 and rel_frob <= 5e-3.
"""
import numpy as np
import torch

from linear_attention_ttt_b200 import ops, synth

TOL_F32 = 1e-4
TOL_BF16_ROW = 2e-2
TOL_BF16_FROB = 5e-3


def max_row_rel(g, o):
    g = np.asarray(g, np.float64).reshape(-1, np.shape(o)[-1])
    o = np.asarray(o, np.float64).reshape(-1, np.shape(o)[-1])
    den = np.max(np.abs(o), axis=1)
    num = np.max(np.abs(g - o), axis=1)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(num / den)) if len(num) else 0.0


def rel_frob(g, o):
    o = np.asarray(o, np.float64)
    n = np.linalg.norm(o)
    return float(np.linalg.norm(np.asarray(g, np.float64) - o) / (n if n > 0 else 1.0))


def check(g, o, dtype, what=""):
    r, f = max_row_rel(g, o), rel_frob(g, o)
    if dtype == synth.F32:
        assert r <= TOL_F32, f"{what}: max_row_rel {r:.3e} > {TOL_F32}"
    else:
        assert r <= TOL_BF16_ROW, f"{what}: max_row_rel {r:.3e} > {TOL_BF16_ROW}"
        assert f <= TOL_BF16_FROB, f"{what}: rel_frob {f:.3e} > {TOL_BF16_FROB}"
    return r, f


def dev(x, dtype, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
    return t.to(torch.bfloat16) if dtype == synth.BF16 else t


def upload_linear(w, device="cuda"):
    return dict(q=dev(w.q, w.dtype, device), k=dev(w.k, w.dtype, device),
                v=dev(w.v, w.dtype, device), eta=dev(w.eta, synth.F32, device),
                W0=dev(w.W0, synth.F32, device))


def run_linear(w, device="cuda", tensors=None):
    t = tensors or upload_linear(w, device)
    out, Wf = ops.ttt_linear_fwd(t["q"], t["k"], t["v"], t["eta"], t["W0"], w.chunk, w.loss)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return out.float().cpu().numpy().astype(np.float64), Wf.cpu().numpy().astype(np.float64)


def upload_lact(w, device="cuda"):
    return dict(q=dev(w.q, w.dtype, device), k=dev(w.k, w.dtype, device),
                v=dev(w.v, w.dtype, device), eta=dev(w.eta, synth.F32, device),
                W1=dev(w.W1, synth.F32, device), W2=dev(w.W2, synth.F32, device),
                W3=dev(w.W3, synth.F32, device))


def run_lact(w, device="cuda", tensors=None):
    t = tensors or upload_lact(w, device)
    out, F1, F2, F3 = ops.lact_swiglu_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                          t["W3"], w.chunk, w.update_rule, w.causal, finals=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    f = lambda x: x.float().cpu().numpy().astype(np.float64)
    return f(out), f(F1), f(F2), f(F3)
