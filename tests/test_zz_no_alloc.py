"""The LaCT entry point that allocates no device memory.

lact_swiglu_fwd_noalloc runs the same layer as lact_swiglu_fwd_ex but keeps
its scratch in a fixed array inside the library instead of allocating it. It
is meant for callers that cannot allocate during the call: engines whose own
allocator already holds almost all of the GPU's memory (an allocation from
this library would fail or fragment it), and latency-critical loops that must
contain no allocation. These tests call it through the C ABI twice in a row,
on two differently sized problems (so the second call runs on whatever the
first left in the shared array), and compare each result with the allocating
entry point within the bf16 tolerances used for this layer. This file is
collected last so that a failure here never hides the other tests.
"""
import pytest
import torch

from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, upload_lact

pytestmark = pytest.mark.gpu


def _both(w):
    t = upload_lact(w)
    args = (t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"], w.chunk,
            w.update_rule, w.causal)
    ref = ops.lact_swiglu_fwd(*args, finals=True)
    got = ops.lact_swiglu_fwd_noalloc(*args, finals=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return [x.float().cpu().numpy() for x in ref], [x.float().cpu().numpy() for x in got]


def test_no_alloc_entry_matches_allocating_entry_on_two_calls():
    cases = [synth.make_lact(1, 2, 512, 128, 256, 128, synth.UPDATE_GD, seed=21, eta_scale=0.02),
             synth.make_lact(2, 1, 640, 64, 256, 256, synth.UPDATE_MUON, seed=22)]
    for w in cases:
        ref, got = _both(w)
        for g, r, name in zip(got, ref, ("y", "W1_final", "W2_final", "W3_final")):
            check(g, r, w.dtype, f"no-alloc vs allocating, {name}")


def test_no_alloc_entry_rejects_problems_larger_than_its_pool():
    w = synth.make_lact(2, 4, 4096, 256, 512, 2048, synth.UPDATE_GD, seed=23)
    t = upload_lact(w)
    with pytest.raises(ops.TTTError) as e:
        ops.lact_swiglu_fwd_noalloc(t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"],
                                    w.chunk)
    assert e.value.code == -10
