"""Benchmark of the chunked TTT-layer forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 5] [--also 2,3,3:256,4]
                    [--impl ours|reference]

A step is one forward pass of the layer over one batch of synthetic inputs
(seeded, shaped like the pages' workloads; see linear_attention_ttt_b200.synth).
Headline workload (the JSON line's own value): LaCT SwiGLU with the Muon
update, batch 1, 8 heads, T=131072, d=128, hidden 512, chunk 4096, bf16
tokens, fp32 fast weights -- the largest single-GPU workload. The same run
also measures the inner-product layer (B4 H16 T4096 d128 b64), small-chunk
TTT-Linear MSE (B8 H16 T8192 d64, chunks 16 and 256) and LaCT GD (B2 H4
T32768 d256 dh512 b2048) and reports them under "workloads" (--also).

Multi-GPU: one process per GPU (torchrun). (batch, head) pairs are
independent, so every rank runs its own replica of the workload with no
collective on the data path (weak scaling); timing is the max over ranks.

Timing: W untimed warm-up steps, then K steps, each between CUDA events on
the launching stream, bracketed by a barrier and device synchronisation.
Before every step L2 is flushed by reading a 256 MB buffer (outside the
events): the read evicts the previous step's lines and writes back its dirty
ones, so no write-back of earlier work lands inside a timed step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from linear_attention_ttt_b200 import ops, synth  # noqa: E402

METRIC = "TTT-layer tokens/s on 1 B200; % of bf16 tensor peak or HBM GB/s roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FMA peak from the unit counts: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["_source"] = "measured"
        return p
    p = dict(FALLBACK_PEAKS)
    p["_source"] = "fallback"
    return p


# ---------------------------------------------------------------------------
# Workload accounting (algorithmic bytes / flops per step)
# ---------------------------------------------------------------------------

def linear_bytes(w):
    es = 2 if w.dtype == synth.BF16 else 4
    per_head_token = (2 * w.dk + 2 * w.dv) * es + 4        # q, k, v in, y out, eta
    state = w.dk * w.dv * 4 * 2                             # W0 read + W_final write
    return w.B * w.H * (w.T * per_head_token + state)


def linear_bwd_flops(w):
    # The token-by-token chain rule: dq = dy W_t^T, the W_t update, R += q^T dy,
    # k R and R e^T at 2 dk dv each, plus for MSE e = k W_s - v, de W_s^T and
    # k^T de: 16 dk dv per head-token (MSE), 10 dk dv (inner product).
    n = 16 if w.loss == synth.LOSS_MSE else 10
    return w.B * w.H * w.T * n * w.dk * w.dv


def ttt_mlp_flops(B, H, T, dk, dv, dh):
    # The per-token rule: h = W1 k, z = W1 q and the W1 update at 2 dk dh each;
    # r = W2 a, g = W2^T r, y = W2 a' and the W2 update at 2 dh dv each.
    return B * H * T * (6 * dk * dh + 8 * dh * dv)


def linear_flops(w):
    # qW, kW and K^T(NE) at 2 dk dv each (MSE) or qW and K^T(NV) (inner
    # product), plus the causal half of the intra-chunk products.
    n_w = 3 if w.loss == synth.LOSS_MSE else 2
    intra = (w.chunk + 1) * (w.dk + w.dv)
    return w.B * w.H * w.T * (n_w * 2 * w.dk * w.dv + intra)


def lact_flops(w):
    per_tok = 18 * w.dk * w.dh  # apply 6 d dh, key fwd 4 d dh, backprop 8 d dh (d = dk = dv)
    f = w.B * w.H * w.T * per_tok
    if w.update_rule == synth.UPDATE_MUON:
        nchunks = (w.T + w.chunk - 1) // w.chunk
        m, n = max(w.dh, w.dk), min(w.dh, w.dk)
        ns = 5 * (2 * 2 * m * n * n + 2 * n ** 3)
        f += w.B * w.H * nchunks * 3 * ns
    return f


def lact_bytes(w):
    es = 2 if w.dtype == synth.BF16 else 4
    return w.B * w.H * w.T * (4 * w.dk * es + 4)


# ---------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, falling back to nvidia-smi)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append(mhz)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                return
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# Runners
# ---------------------------------------------------------------------------

def upload(w, device):
    def t(x, dtype):
        a = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        a = a.to(device)
        return a.to(torch.bfloat16) if dtype == synth.BF16 else a
    d = {"q": t(w.q, w.dtype), "k": t(w.k, w.dtype), "v": t(w.v, w.dtype),
         "eta": t(w.eta, synth.F32)}
    if w.variant == "lact":
        d.update(W1=t(w.W1, synth.F32), W2=t(w.W2, synth.F32), W3=t(w.W3, synth.F32))
    else:
        d["W0"] = t(w.W0, synth.F32)
    return d


class Step:
    """One forward of the layer on resident device tensors (outputs preallocated)."""

    def __init__(self, w, d):
        self.w, self.d = w, d
        dt = d["q"].dtype
        self.out = torch.empty((w.B, w.H, w.T, w.dv), dtype=dt, device=d["q"].device)
        if w.variant == "lact":
            # prep rows kernel, then per chunk two GEMM launches and the rows
            # kernel (+ Newton-Schulz for Muon, + two apply GEMMs when non-causal)
            nch = -(-w.T // w.chunk) if w.T > 0 else 0
            per = 3 + (1 if w.update_rule == synth.UPDATE_MUON else 0) + (0 if w.causal else 2)
            self.launches = 1 + nch * per
        else:
            self.Wf = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=d["q"].device)
            self.launches = 1

    def __call__(self):
        w, d = self.w, self.d
        if w.variant == "lact":
            ops.lact_swiglu_fwd(d["q"], d["k"], d["v"], d["eta"], d["W1"], d["W2"], d["W3"],
                                w.chunk, w.update_rule, w.causal, out=self.out)
        else:
            ops.ttt_linear_fwd(d["q"], d["k"], d["v"], d["eta"], d["W0"], w.chunk, w.loss,
                               out=self.out, W_final=self.Wf)


def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key, sha):
    """DRAM bytes per launch from a committed ncu capture, if taken on this
    exact kernel source (profiles/traffic.json)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel_key)
    if not rec or rec.get("source_sha") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


KERNEL_SOURCES = {
    "la_tc": ["linear_attention_ttt_b200/csrc/la_tc.cu",
              "linear_attention_ttt_b200/csrc/common.cuh",
              "linear_attention_ttt_b200/csrc/tma.cuh",
              "linear_attention_ttt_b200/csrc/umma.cuh"],
    "ttt_linear_bf16": ["linear_attention_ttt_b200/csrc/ttt_linear_bf16.cu",
                        "linear_attention_ttt_b200/csrc/common.cuh",
                        "linear_attention_ttt_b200/csrc/tma.cuh"],
    "ttt_linear_f32": ["linear_attention_ttt_b200/csrc/ttt_linear_f32.cu",
                       "linear_attention_ttt_b200/csrc/common.cuh"],
    "ttt_linear_wy": ["linear_attention_ttt_b200/csrc/ttt_linear_wy.cu",
                      "linear_attention_ttt_b200/csrc/common.cuh",
                      "linear_attention_ttt_b200/csrc/tma.cuh"],
}


def kernel_key(w):
    if w.variant == "lact":
        return "lact"
    if w.dtype != synth.BF16:
        return "ttt_linear_f32"
    if w.loss == synth.LOSS_NEG_DOT and w.dk == 128 and w.dv == 128:
        return "la_tc"
    if (w.loss == synth.LOSS_MSE and w.dk == 64 and w.dv == 64
            and (w.chunk in (16, 32) or w.chunk % 64 == 0)):
        return "ttt_linear_wy"
    return "ttt_linear_bf16"


def rank_workload(index, rank, chunk=None, seq_len=None):
    """Each rank runs its own replica: the same workload shape with an
    independent draw of the inputs (weak scaling, no data-path collective).
    seq_len shortens the sequence (same distributions), e.g. for profiling."""
    return synth.config(index, chunk=chunk, T=seq_len, replica=rank)


def max_over_ranks(value, dist=None, device=None):
    """Max of a per-rank scalar over all ranks (a float on every rank)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step, world, ms_per_step):
    """Whole-job tokens/s: every rank processed tokens_per_step per step and
    the job's step time is the slowest rank's."""
    return tokens_per_step * world / (ms_per_step / 1e3)


def cpu_oracle_step(w, sample_heads):
    """Runs the fp64 oracle on the first `sample_heads` (batch, head)
    sequences of the workload (all of them for sample_heads >= B*H); returns
    (seconds, tokens) with tokens counted in the metric's unit (batch rows x T:
    one (batch, head) sequence is 1/H of a batch row)."""
    from oracle import ttt_oracle as O
    n = min(sample_heads, w.B * w.H)
    nb, nh = (n // w.H, w.H) if n >= w.H else (1, n)
    sl = (slice(0, nb), slice(0, nh))
    t0 = time.perf_counter()
    if w.variant == "lact":
        O.lact_swiglu(w.q[sl], w.k[sl], w.v[sl], w.eta[sl], w.W1[:nh], w.W2[:nh], w.W3[:nh],
                      w.chunk, w.update_rule, w.causal)
    else:
        W0 = w.W0[:nh] if w.W0.ndim == 3 else w.W0[sl]
        O.ttt_linear_dual(w.q[sl], w.k[sl], w.v[sl], w.eta[sl], W0, w.chunk, w.loss)
    dt = time.perf_counter() - t0
    return dt, w.T * nb * nh / w.H


def cpu_sample_heads(w):
    """All sequences for TTT-Linear workloads (a few seconds of fp64 work);
    two sequences for LaCT (each costs tens of GFLOP in fp64)."""
    return w.B * w.H if w.variant != "lact" else 2


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def parse_extra(spec):
    """'2,3,3:256,4' -> [(2, None), (3, None), (3, 256), (4, None)]"""
    out = []
    for item in filter(None, (x.strip() for x in spec.split(","))):
        idx, _, ch = item.partition(":")
        out.append((int(idx), int(ch) if ch else None))
    return out


def roofline(w, ms_per_launch, pk):
    """Roofline entry of the kernel (TTT-Linear: the one launch of a step) or
    of the whole step (LaCT: every launch of the chunk loop, so the figure is
    a lower bound on the GEMM kernel's own fraction)."""
    key = kernel_key(w)
    if w.variant == "lact":
        flops = lact_flops(w)
        peak = pk["bf16_tflops"]
        achieved = flops / (ms_per_launch / 1e3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None,
                "peak_source": pk["_source"] + " bf16_tflops (burst: a step of a few ms timed alone)",
                "kernel": "lact step (all launches)", "algorithmic_flops_per_step": flops}
    byts = linear_bytes(w)
    achieved = byts / (ms_per_launch / 1e3) / 1e9
    sha = source_sha(KERNEL_SOURCES[key])
    return {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "traffic": recorded_traffic(key, sha),
            "peak_source": pk["_source"] + " hbm_gbs", "kernel": key,
            "algorithmic_bytes_per_launch": byts, "kernel_source_sha": sha}


def cpu_baseline(w):
    n = cpu_sample_heads(w)
    dt, toks = cpu_oracle_step(w, n)
    return {"value": toks / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle (dual form / LaCT scan) on {n} of {w.B * w.H} "
                      f"(batch, head) sequences, {dt:.1f} s"}


def workload_cfg(w, world):
    cfg = {"workload": w.name, "batch": w.B, "heads": w.H, "seq_len": w.T, "dk": w.dk,
           "dv": w.dv, "chunk": w.chunk, "variant": w.variant,
           "loss": ("mse" if w.loss == 0 else "neg_dot") if w.variant != "lact" else "neg_dot_swiglu",
           "parallelism": f"replicas{world}"}
    if w.variant == "lact":
        cfg.update(dh=w.dh, update_rule="muon" if w.update_rule else "gd", causal=w.causal)
    return cfg


class Runner:
    """Times workloads on this rank's GPU (device-resident inputs; CUDA events
    on the launching stream; L2 flushed by a read before every timed step)."""

    def __init__(self, args, dist, device):
        self.args, self.dist, self.device = args, dist, device
        # 256 MB > L2: reading it evicts every line the previous step left,
        # and dirty lines are written back during the read, outside the timing.
        self.flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
        self.stream = torch.cuda.current_stream()

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def l2_flush(self):
        torch.sum(self.flush)

    def device_timing(self, step):
        args = self.args
        nvtx = torch.cuda.nvtx  # named ranges for profilers (no effect without one)
        nvtx.range_push("warmup")
        for _ in range(args.warmup):
            self.l2_flush()
            step()
        torch.cuda.synchronize()
        nvtx.range_pop()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        self.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(self.device.index)
        with sampler:
            nvtx.range_push("timed")
            t_wall = time.perf_counter()
            for i in range(args.steps):
                self.l2_flush()
                ev[i][0].record(self.stream)
                step()
                ev[i][1].record(self.stream)
            torch.cuda.synchronize()
            t_wall = time.perf_counter() - t_wall
            nvtx.range_pop()
        self.barrier()
        per = [a.elapsed_time(b) for a, b in ev]
        ms = max_over_ranks(sum(per), self.dist, self.device) / args.steps
        return ms, sampler.summary(), t_wall

    def e2e(self, w, d, step):
        """Same metric through the public API with host buffers, as a stream of
        steps: every step copies its inputs from pinned host memory to the
        device and reads its results back (y, and W_final for TTT-Linear),
        all inside the timed region. Two device buffer sets let the upload of
        one step and the read-back of another run on two copy streams while a
        third step computes, so the step time is bounded by the slowest of
        the three rather than their sum."""
        host = {k: v.to("cpu").pin_memory() for k, v in d.items()}
        d2 = {k: torch.empty_like(v) for k, v in d.items()}
        sets = [(d, step), (d2, Step(w, d2))]

        def results(st):
            return [st.out] + ([st.Wf] if getattr(st, "Wf", None) is not None else [])
        host_res = [[torch.empty(r.shape, dtype=r.dtype).pin_memory() for r in results(st)]
                    for _, st in sets]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(r.numel() * r.element_size() for r in host_res[0])
        n = max(3, min(self.args.steps, 20))
        comp = self.stream
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def one(i):
            b = i % 2
            dd, st = sets[b]
            s_in.wait_event(ev_comp[b])          # the last step on this set has read its inputs
            with torch.cuda.stream(s_in):
                for k2, v2 in host.items():
                    dd[k2].copy_(v2, non_blocking=True)
            ev_in[b].record(s_in)
            comp.wait_event(ev_in[b])
            comp.wait_event(ev_out[b])          # and its results have been read back
            with torch.cuda.stream(comp):
                st()
            ev_comp[b].record(comp)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                for hr, r in zip(host_res[b], results(st)):
                    hr.copy_(r, non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(2):
            one(i)
        torch.cuda.synchronize()
        self.barrier()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("e2e")
        a.record(comp)
        s_in.wait_event(a)
        s_out.wait_event(a)
        for i in range(n):
            one(i)
        comp.wait_event(ev_out[0])
        comp.wait_event(ev_out[1])
        e.record(comp)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        ms = max_over_ranks(a.elapsed_time(e) / n, self.dist, self.device)
        del sets, d2
        return ms, h2d, d2h

    def measure(self, w, world, with_e2e):
        d = upload(w, self.device)
        step = Step(w, d)
        ms, clocks, t_wall = self.device_timing(step)
        res = {"ms_per_step": ms, "value": job_throughput(w.B * w.T, world, ms),
               "roofline": roofline(w, ms, peaks()),
               "gpu_launches": (step.launches or 0) * self.args.steps,
               "clocks": clocks, "wall_s_timed": t_wall}
        if with_e2e:
            e_ms, h2d, d2h = self.e2e(w, d, step)
            res["e2e"] = {"value": job_throughput(w.B * w.T, world, e_ms), "unit": "tokens/s",
                          "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world}
        del step, d
        torch.cuda.empty_cache()
        return res


def window_flops(B, H, T, d, window):
    """QK^T and PV over the causal window: 4 d flops per (query, key) pair."""
    pairs = sum(min(t + 1, window) for t in range(T)) if T <= 1 << 16 else (
        window * (window + 1) // 2 + (T - window) * window if T > window else T * (T + 1) // 2)
    return 4 * d * B * H * pairs


def measure_next_rows(runner, device):
    """The scope table's next rows, each timed like the hot path (device
    events over K steps after W warm-ups, L2 flushed by a read before every
    step) on synthetic inputs of the pages' shapes. Returns a list of dicts."""
    from linear_attention_ttt_b200 import cp  # noqa: F401  (binding of the context-parallel call)
    pk = peaks()
    out = []

    def dev(x, dtype):
        a = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
        return a.to(torch.bfloat16) if dtype == synth.BF16 else a

    def run(row, cfg, step, tokens, roof=None, launches=None):
        ms, clocks, _ = runner.device_timing(step)
        item = {"row": row, "config": cfg, "ms_per_step": ms, "value": tokens / (ms / 1e3),
                "unit": "tokens/s", "clocks": clocks}
        if roof is not None:
            kind, work, peak, unit, kernel = roof
            ach = work / (ms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
            item["roofline"] = {"bound": kind, "achieved": ach, "peak": peak, "unit": unit,
                                "frac": ach / peak, "kernel": kernel,
                                "peak_source": ("fp32 FMA lanes x max SM clock (derived)"
                                                if kind == "alu" else pk["_source"])}
        out.append(item)
        torch.cuda.empty_cache()

    # f1: TTT-Linear MSE / inner-product backward, at the forward workloads' sizes
    for idx in (3, 2):
        w = synth.config(idx)
        T = w.T
        t = {n: dev(getattr(w, n), w.dtype if n in "qkv" else synth.F32)
             for n in ("q", "k", "v", "eta", "W0")}
        dy = torch.randn_like(t["v"])
        run(f"f1 backward {'mse' if w.loss == 0 else 'inner product'}",
            {"workload": w.name, "batch": w.B, "heads": w.H, "seq_len": T, "d": w.dk,
             "chunk": w.chunk},
            lambda: ops.ttt_linear_bwd(t["q"], t["k"], t["v"], t["eta"], t["W0"], w.chunk,
                                       w.loss, dy), w.B * T,
            roof=("alu", linear_bwd_flops(w), FP32_ALU_TFLOPS, "TFLOP/s", "ttt_linear_bwd"))
        del t, dy
    # f1: LaCT backward (GD), one shortened head pair of the d = 128 shape
    w = synth.make_lact(1, 2, 4096, 128, 512, 1024, synth.UPDATE_GD, seed=1090)
    t = {n: dev(getattr(w, n), w.dtype if n in "qkv" else synth.F32)
         for n in ("q", "k", "v", "eta", "W1", "W2", "W3")}
    dy = torch.randn_like(t["v"])
    run("f1 backward lact gd", {"workload": "lact_bwd_B1_H2_T4096_d128_dh512_b1024"},
        lambda: ops.lact_swiglu_bwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"],
                                    w.chunk, 0, 1, dy), w.B * w.T)
    del t, dy
    # f2: LaCT momentum at the GD workload's size
    w = synth.config(4)
    t = {n: dev(getattr(w, n), w.dtype if n in "qkv" else synth.F32)
         for n in ("q", "k", "v", "eta", "W1", "W2", "W3")}
    o = torch.empty_like(t["v"])
    run("f2 momentum (beta 0.9)", {"workload": w.name + "_momentum"},
        lambda: ops.lact_swiglu_fwd_momentum(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                             t["W3"], w.chunk, 0.9, out=o), w.B * w.T,
        ("tensor", lact_flops(w), pk["bf16_tflops"], "TFLOP/s", "lact step (all launches)"))
    # f4b: context-parallel call with no exchange (one rank) at the same size
    run("f4b context parallel (1 rank)", {"workload": w.name + "_cp1"},
        lambda: cp.lact_swiglu_fwd_cp(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                      t["W3"], w.chunk, 0, None, out=o), w.B * w.T,
        ("tensor", lact_flops(w), pk["bf16_tflops"], "TFLOP/s", "lact step (all launches)"))
    del t, o
    # f3: TTT-MLP, head 64, hidden 256, chunk 16
    w = synth.config(3, B=4, T=2048)
    rng = np.random.default_rng(7)
    P = [rng.standard_normal((w.H, 256, 64)) / 8, np.zeros((w.H, 256)),
         rng.standard_normal((w.H, 64, 256)) / 16, np.zeros((w.H, 64))]
    t = [dev(getattr(w, n), w.dtype) for n in ("q", "k", "v")] + [dev(w.eta, synth.F32)]
    Pd = [dev(p, synth.F32) for p in P]
    run("f3 ttt-mlp", {"workload": "ttt_mlp_bf16_B4_H16_T2048_d64_dh256_b16"},
        lambda: ops.ttt_mlp_fwd(*t, *Pd, 16), w.B * w.T,
        roof=("alu", ttt_mlp_flops(w.B, w.H, w.T, w.dk, w.dv, 256), FP32_ALU_TFLOPS, "TFLOP/s",
              "ttt_mlp"))
    del t, Pd
    # f4a: window attention (window 4096) and the LaCT + window block, Muon workload
    w = synth.config(5)
    t = {n: dev(getattr(w, n), w.dtype if n in "qkv" else synth.F32)
         for n in ("q", "k", "v", "eta", "W1", "W2", "W3")}
    o = torch.empty_like(t["v"])
    wf = window_flops(w.B, w.H, w.T, w.dk, 4096)
    run("f4a window attention (w 4096)", {"workload": w.name + "_window4096"},
        lambda: ops.window_attention_fwd(t["q"], t["k"], t["v"], 4096, out=o), w.B * w.T,
        ("tensor", wf, pk["bf16_tflops"], "TFLOP/s", "window_attn_kernel"))
    run("f4a lact + window attention", {"workload": w.name + "_lact_window4096"},
        lambda: ops.lact_swiglu_window_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"],
                                           t["W3"], w.chunk, w.update_rule, 4096, out=o),
        w.B * w.T,
        ("tensor", wf + lact_flops(w), pk["bf16_tflops"], "TFLOP/s", "lact step + window"))
    del t, o
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=5,
                    help="headline workload (default 5: LaCT Muon, the largest single-GPU one)")
    ap.add_argument("--chunk", type=int, default=None)
    ap.add_argument("--also", default="2,3,3:256,4",
                    help="workloads measured in the same run and reported under 'workloads' "
                         "(index[:chunk], comma separated; '' for none)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="shorter sequence of the same workload (profiling); the default "
                         "line uses the workload's own length")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip timing the next rows (backward, momentum, TTT-MLP, window "
                         "attention, context parallelism), reported under 'next_rows'")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    w = rank_workload(args.workload, rank, chunk=args.chunk, seq_len=args.seq_len)
    base_cfg = workload_cfg(w, world)

    if args.impl == "reference":
        if rank != 0:
            return
        steps = []
        sample_heads = max(1, cpu_sample_heads(w) // 4)
        for i in range(args.warmup + args.steps):
            dt, toks = cpu_oracle_step(w, sample_heads)
            if i >= args.warmup:
                steps.append(toks / dt)
        v = float(statistics.median(steps))
        sample = f"fp64 numpy oracle on {sample_heads} (batch, head) sequence(s) of the workload per step"
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
                "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "dtype": "f64", "data": "synthetic",
                "config": base_cfg,
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(),
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    ops.load()
    runner = Runner(args, dist, device)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline

    head = runner.measure(w, world, with_e2e=True)
    cfg = dict(base_cfg)
    cfg["l2"] = "flushed before every timed step (256 MB read, outside the timed events)"
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == synth.BF16 else "f32", "data": "synthetic",
            "config": cfg, "roofline": head["roofline"], "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
            "wall_s_timed": head["wall_s_timed"]}
    if want_cpu:
        line["cpu_baseline"] = cpu_baseline(w)

    extras = []
    for idx, ch in parse_extra(args.also):
        wx = rank_workload(idx, rank, chunk=ch, seq_len=args.seq_len)
        r = runner.measure(wx, world, with_e2e=False)
        item = {"config": workload_cfg(wx, world), "ms_per_step": r["ms_per_step"],
                "value": r["value"], "unit": "tokens/s",
                "dtype": "bf16" if wx.dtype == synth.BF16 else "f32",
                "roofline": r["roofline"], "gpu_launches": r["gpu_launches"],
                "clocks": r["clocks"]}
        if want_cpu:
            item["cpu_baseline"] = cpu_baseline(wx)
        extras.append(item)
        del wx
    if extras:
        line["workloads"] = extras
        line["gpu_launches"] += sum(x["gpu_launches"] for x in extras)
    if not args.no_next_rows:
        line["next_rows"] = measure_next_rows(runner, device)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
