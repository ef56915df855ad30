"""bench.py's accounting, checked on the CPU: the algorithmic bytes and flops
behind roofline.achieved, the kernel each workload is attributed to, and the
whole-job throughput."""
import numpy as np
import pytest

import bench
from linear_attention_ttt_b200 import synth


@pytest.mark.parametrize("index", [1, 2, 3])
def test_linear_bytes_are_the_tensors_read_and_written(index):
    w = synth.config(index, T=128)
    es = 2 if w.dtype == synth.BF16 else 4
    tokens = (w.q.size + w.k.size + w.v.size) * es          # inputs
    out = w.B * w.H * w.T * w.dv * es                       # y
    eta = w.eta.size * 4
    state = 2 * w.B * w.H * w.dk * w.dv * 4                 # W0 read, W_final written
    assert bench.linear_bytes(w) == tokens + out + eta + state


def gemm(m, n, k):
    return 2 * m * n * k


@pytest.mark.parametrize("index", [4, 5])
def test_lact_flops_count_every_product(index):
    w = synth.config(index, T=2 * synth.config(index, T=64).chunk)
    d, dh, b = w.dk, w.dh, w.chunk
    per_chunk = (gemm(b, dh, d) * 2 + gemm(b, d, dh)          # apply: Q W1^T, Q W3^T, Aq W2^T
                 + gemm(b, dh, d) * 2                         # key side: K W1^T, K W3^T
                 + gemm(b, dh, d)                             # Gz = -eta V W2
                 + gemm(d, dh, b)                             # G2 = -V~^T Ak
                 + gemm(dh, d, b) * 2)                        # G1 = dH1^T K, G3 = dH3^T K
    nchunks = w.T // b
    want = w.B * w.H * nchunks * per_chunk
    if w.update_rule == synth.UPDATE_MUON:
        m, n = max(dh, d), min(dh, d)
        per_ns_step = gemm(n, n, m) + gemm(n, n, n) + gemm(m, n, n)   # Gram, its square, X (bA + cA^2)
        want += w.B * w.H * nchunks * 3 * 5 * per_ns_step
    assert bench.lact_flops(w) == want


@pytest.mark.parametrize("index,key", [(1, "ttt_linear_f32"), (2, "la_tc"), (3, "ttt_linear_wy"),
                                       (4, "lact"), (5, "lact")])
def test_workloads_are_attributed_to_the_kernel_that_runs_them(index, key):
    assert bench.kernel_key(synth.config(index, T=64)) == key
    assert bench.kernel_key(synth.config(3, chunk=24, T=64)) == "ttt_linear_bf16"
    assert bench.kernel_key(synth.config(3, chunk=256, T=64)) == "ttt_linear_wy"


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1000, 4, 2.0) == pytest.approx(2e6)
    assert bench.job_throughput(1000, 1, 0.5) == pytest.approx(2e6)


def test_kernel_sources_exist_and_hash():
    for key, paths in bench.KERNEL_SOURCES.items():
        sha = bench.source_sha(paths)
        assert len(sha) == 16 and int(sha, 16) >= 0
