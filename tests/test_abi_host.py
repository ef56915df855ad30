"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/ttt.h declares, and rejects bad arguments before any
CUDA call. Descriptors carry fake (aligned, never dereferenced) pointers."""
import ctypes
import os
import re

import pytest

from linear_attention_ttt_b200 import build as B
from linear_attention_ttt_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttt.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ops.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"^\s*typedef[^;]*;", "", text, flags=re.M | re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("ttt_linear_fwd", "lact_swiglu_fwd", "lact_swiglu_fwd_ex", "ttt_status_string",
              "ttt_get_device_status", "ttt_version", "ttt_linear_bwd", "lact_swiglu_fwd_momentum",
              "ttt_mlp_fwd", "window_attention_fwd", "lact_swiglu_window_fwd",
              "lact_swiglu_fwd_cp", "lact_swiglu_fwd_noalloc", "ttt_test_fail_allocations"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert lib.ttt_version() >= 100
    assert lib.ttt_status_string(-5).decode().startswith("no kernel")


FAKE = 1 << 32  # 16-byte aligned, never dereferenced


def tok(B, H, T, d, dtype=ops.TTT_BF16, base=FAKE, strides=None):
    t = ops.TTTTensor()
    t.data, t.dtype, t.ndim = base, dtype, 4
    for i, s in enumerate((B, H, T, d)):
        t.shape[i] = s
    st = strides or (H * T * d, T * d, d, 1)
    for i, s in enumerate(st):
        t.stride[i] = s
    return t


def dense(shape, base, dtype=ops.TTT_F32):
    t = ops.TTTTensor()
    t.data, t.dtype, t.ndim = base, dtype, len(shape)
    s = 1
    for i in reversed(range(len(shape))):
        t.shape[i] = shape[i]
        t.stride[i] = s
        s *= shape[i]
    return t


class Case:
    """A valid ttt_linear_fwd call whose fields tests break one at a time."""

    def __init__(self, B=2, H=3, T=40, dk=64, dv=64, dtype=ops.TTT_BF16):
        gap = 1 << 28
        self.q = tok(B, H, T, dk, dtype, FAKE)
        self.k = tok(B, H, T, dk, dtype, FAKE + gap)
        self.v = tok(B, H, T, dv, dtype, FAKE + 2 * gap)
        self.eta = dense((B, H, T), FAKE + 3 * gap)
        self.W0 = dense((H, dk, dv), FAKE + 4 * gap)
        self.out = tok(B, H, T, dv, dtype, FAKE + 5 * gap)
        self.Wf = dense((B, H, dk, dv), FAKE + 6 * gap)
        self.chunk, self.loss = 16, ops.TTT_LOSS_MSE

    def call(self, lib):
        r = ctypes.byref
        return lib.ttt_linear_fwd(r(self.q), r(self.k), r(self.v), r(self.eta), r(self.W0),
                                  self.chunk, self.loss, r(self.out),
                                  r(self.Wf) if self.Wf is not None else None, None)


ERR = {k: v for v, k in ops.STATUS.items()}


def test_rejects_bad_scalars(lib):
    c = Case()
    c.chunk = 0
    assert c.call(lib) == ERR["TTT_ERR_ARG"]
    c = Case()
    c.loss = 7
    assert c.call(lib) == ERR["TTT_ERR_ARG"]


def test_rejects_null(lib):
    c = Case()
    assert lib.ttt_linear_fwd(None, ctypes.byref(c.k), ctypes.byref(c.v), ctypes.byref(c.eta),
                              ctypes.byref(c.W0), 16, 0, ctypes.byref(c.out), None, None) \
        == ERR["TTT_ERR_NULL"]
    c.Wf.data = 0
    assert c.call(lib) == ERR["TTT_ERR_NULL"]


def test_rejects_shape_mismatch(lib):
    c = Case()
    c.k.shape[2] = 41
    assert c.call(lib) == ERR["TTT_ERR_SHAPE"]
    c = Case()
    c.W0 = dense((3, 64, 32), c.W0.data)
    assert c.call(lib) == ERR["TTT_ERR_SHAPE"]
    c = Case()
    c.eta = dense((2, 3, 39), c.eta.data)
    assert c.call(lib) == ERR["TTT_ERR_SHAPE"]
    c = Case()
    c.out.ndim = 3
    assert c.call(lib) == ERR["TTT_ERR_SHAPE"]


def test_rejects_dtype_mismatch(lib):
    c = Case()
    c.v.dtype = ops.TTT_F32
    assert c.call(lib) == ERR["TTT_ERR_DTYPE"]
    c = Case()
    c.eta.dtype = ops.TTT_BF16
    assert c.call(lib) == ERR["TTT_ERR_DTYPE"]
    c = Case()
    c.W0.dtype = ops.TTT_BF16
    assert c.call(lib) == ERR["TTT_ERR_DTYPE"]


def test_rejects_layout_violations(lib):
    c = Case()
    c.q.stride[3] = 2
    assert c.call(lib) == ERR["TTT_ERR_LAYOUT"]
    c = Case()
    c.k.data += 8  # not 16-byte aligned
    assert c.call(lib) == ERR["TTT_ERR_LAYOUT"]
    c = Case(dk=60, dv=60)  # token stride of 120 bytes is not a multiple of 16
    assert c.call(lib) == ERR["TTT_ERR_LAYOUT"]
    c = Case()
    c.W0.stride[2] = 2  # not contiguous
    assert c.call(lib) == ERR["TTT_ERR_LAYOUT"]


def test_rejects_output_overlapping_an_input(lib):
    c = Case()
    c.out.data = c.v.data
    assert c.call(lib) == ERR["TTT_ERR_ARG"]
    c = Case()
    c.Wf.data = c.W0.data
    assert c.call(lib) == ERR["TTT_ERR_ARG"]


def test_rejects_oversized_heads(lib):
    c = Case(dk=512, dv=512)
    assert c.call(lib) == ERR["TTT_ERR_UNSUPPORTED"]


def test_rejects_sizes_beyond_32_bit_indexing(lib):
    """More than 2^30 tokens or 2^24 (batch, head) pairs: refused before any
    descriptor is read further (the kernels index with 32-bit integers)."""
    c = Case(T=(1 << 30) + 1)
    assert c.call(lib) == ERR["TTT_ERR_UNSUPPORTED"]
    c = Case(B=1 << 12, H=(1 << 12) + 1)
    assert c.call(lib) == ERR["TTT_ERR_UNSUPPORTED"]

    def long_seq(ts):
        T = (1 << 30) + 1
        for n in ("q", "k", "v", "out"):
            ts[n] = tok(1, 2, T, 128, base=ts[n].data)
        ts["eta"] = dense((1, 2, T), ts["eta"].data)
    assert lact_call(lib, mutate=long_seq) == ERR["TTT_ERR_UNSUPPORTED"]
    assert lact_call(lib, dh=8192) == ERR["TTT_ERR_UNSUPPORTED"]


def lact_call(lib, rule=0, causal=1, dh=512, mutate=None):
    gap = 1 << 28
    Bs, H, T, d = 1, 2, 64, 128
    ts = dict(q=tok(Bs, H, T, d, base=FAKE), k=tok(Bs, H, T, d, base=FAKE + gap),
              v=tok(Bs, H, T, d, base=FAKE + 2 * gap), eta=dense((Bs, H, T), FAKE + 3 * gap),
              W1=dense((H, dh, d), FAKE + 4 * gap), W2=dense((H, d, dh), FAKE + 5 * gap),
              W3=dense((H, dh, d), FAKE + 6 * gap), out=tok(Bs, H, T, d, base=FAKE + 7 * gap))
    if mutate:
        mutate(ts)
    r = ctypes.byref
    return lib.lact_swiglu_fwd(r(ts["q"]), r(ts["k"]), r(ts["v"]), r(ts["eta"]), r(ts["W1"]),
                               r(ts["W2"]), r(ts["W3"]), 32, rule, causal, r(ts["out"]), None)


def test_lact_rejects_bad_arguments(lib):
    assert lact_call(lib, rule=3) == ERR["TTT_ERR_ARG"]
    assert lact_call(lib, causal=2) == ERR["TTT_ERR_ARG"]

    def bad_w2(ts):
        ts["W2"] = dense((2, 128, 256), ts["W2"].data)
    assert lact_call(lib, mutate=bad_w2) == ERR["TTT_ERR_SHAPE"]

    def w3_bf16(ts):
        ts["W3"].dtype = ops.TTT_BF16
    assert lact_call(lib, mutate=w3_bf16) == ERR["TTT_ERR_DTYPE"]

    def alias(ts):
        ts["out"].data = ts["q"].data
    assert lact_call(lib, mutate=alias) == ERR["TTT_ERR_ARG"]


def noalloc_call(lib, H, T, d, dh, chunk, rule):
    gap = 1 << 36
    ts = [tok(1, H, T, d, base=FAKE), tok(1, H, T, d, base=FAKE + gap),
          tok(1, H, T, d, base=FAKE + 2 * gap), dense((1, H, T), FAKE + 3 * gap),
          dense((H, dh, d), FAKE + 4 * gap), dense((H, d, dh), FAKE + 5 * gap),
          dense((H, dh, d), FAKE + 6 * gap), tok(1, H, T, d, base=FAKE + 7 * gap)]
    r = ctypes.byref
    return lib.lact_swiglu_fwd_noalloc(*(r(t) for t in ts[:7]), chunk, rule, 1, r(ts[7]),
                                       None, None, None, None)


def documented_scratch_per_pair(d, dh, chunk, T, muon):
    """The per-(batch, head) scratch need as include/ttt.h states it for
    lact_swiglu_fwd_noalloc."""
    E, R, c = 2 * dh * d + d * dh, 2 * dh + d, min(chunk, T)
    need = 4 * (2 * E + R) + 2 * (E + 4 * c * dh) * (2 if muon else 1)
    if muon and not (d == 128 and dh == 512):
        s = min(d, dh)
        need += 4 * 3 * (16 * s * s + dh * d + 64)
    return need


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="fake pointers: on a GPU a call that fits would launch")
@pytest.mark.parametrize("d,dh,chunk,T,rule", [(128, 512, 1024, 4096, 0), (128, 512, 256, 4096, 1),
                                               (64, 256, 512, 2048, 1), (256, 512, 128, 512, 0),
                                               (256, 1024, 64, 100, 1)])
def test_noalloc_scratch_limit_is_the_documented_formula(lib, d, dh, chunk, T, rule):
    """The largest number of (batch, head) pairs the 32 MiB array accepts is
    the one the header's formula (and its worked example) predicts: that many
    pairs pass the size check (and, with no GPU, stop at the CUDA lookup),
    one more returns TTT_ERR_SCRATCH before any CUDA call."""
    per = documented_scratch_per_pair(d, dh, chunk, T, rule == 1)
    n_max = ((32 << 20) - 4096) // per
    if (d, dh, chunk, rule) == (128, 512, 1024, 0):
        assert per == 6164992 and n_max == 5      # the header's worked example
    assert n_max >= 1
    assert noalloc_call(lib, n_max, T, d, dh, chunk, rule) == ERR["TTT_ERR_CUDA"]
    assert noalloc_call(lib, n_max + 1, T, d, dh, chunk, rule) == ERR["TTT_ERR_SCRATCH"]


def momentum_call(lib, beta=0.9, mutate=None):
    gap = 1 << 28
    Bs, H, T, d, dh = 1, 2, 64, 128, 256
    ts = dict(q=tok(Bs, H, T, d, base=FAKE), k=tok(Bs, H, T, d, base=FAKE + gap),
              v=tok(Bs, H, T, d, base=FAKE + 2 * gap), eta=dense((Bs, H, T), FAKE + 3 * gap),
              W1=dense((H, dh, d), FAKE + 4 * gap), W2=dense((H, d, dh), FAKE + 5 * gap),
              W3=dense((H, dh, d), FAKE + 6 * gap), M1=dense((H, dh, d), FAKE + 7 * gap),
              M2=None, M3=None, out=tok(Bs, H, T, d, base=FAKE + 8 * gap),
              M1f=dense((Bs, H, dh, d), FAKE + 9 * gap))
    if mutate:
        mutate(ts)
    r = lambda x: ctypes.byref(x) if x is not None else None
    return lib.lact_swiglu_fwd_momentum(*(r(ts[n]) for n in ("q", "k", "v", "eta", "W1", "W2", "W3")),
                                        32, beta, 1, r(ts["M1"]), r(ts["M2"]), r(ts["M3"]),
                                        r(ts["out"]), None, None, None, r(ts["M1f"]), None, None,
                                        None)


def test_momentum_entry_rejects_bad_arguments(lib):
    beta = float
    assert momentum_call(lib, beta(float("nan"))) == ERR["TTT_ERR_ARG"]
    assert momentum_call(lib, beta(float("inf"))) == ERR["TTT_ERR_ARG"]

    def bad_m1(ts):
        ts["M1"] = dense((2, 128, 256), ts["M1"].data)
    assert momentum_call(lib, beta(0.9), bad_m1) == ERR["TTT_ERR_SHAPE"]

    def m1_bf16(ts):
        ts["M1"].dtype = ops.TTT_BF16
    assert momentum_call(lib, beta(0.9), m1_bf16) == ERR["TTT_ERR_DTYPE"]

    def final_on_input(ts):
        ts["M1f"].data = ts["M1"].data
    assert momentum_call(lib, beta(0.9), final_on_input) == ERR["TTT_ERR_ARG"]

    def final_on_out(ts):
        ts["M1f"].data = ts["out"].data
    assert momentum_call(lib, beta(0.9), final_on_out) == ERR["TTT_ERR_ARG"]
