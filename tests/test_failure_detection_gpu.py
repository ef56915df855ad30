"""Failure detection on the GPU without faulting it: a bounded wait that runs
out is reported through the device status word, and the context stays
usable afterwards."""
import pytest

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, run_linear

pytestmark = pytest.mark.gpu

ERR = {name: code for code, name in ops.STATUS.items()}


def test_bounded_wait_reports_timeout_and_the_context_survives():
    assert ops.device_status() == 0
    ops.selftest_wait_timeout()          # a wait nothing completes (about 2 s)
    assert ops.device_status() == ERR["TTT_ERR_TIMEOUT"]
    assert ops.device_status() == 0      # reading the status cleared it
    w = synth.make_ttt_linear(1, 2, 40, 64, 64, 16, synth.BF16, ops.TTT_LOSS_NEG_DOT, seed=3,
                              eta_kind="softplus", eta_scale=0.05)
    y, Wf = run_linear(w)                # checks the status word is clean again
    yo, Wo = O.ttt_linear_minibatch(w.q, w.k, w.v, w.eta, w.W0, w.chunk, w.loss)
    check(y, yo, w.dtype, "y")
    check(Wf, Wo, w.dtype, "W_final")


def test_failed_scratch_allocation_is_reported_and_recovers():
    """Host-side injection (no GPU fault): the next scratch allocation fails as
    if the device were out of memory. The call returns TTT_ERR_ALLOC, writes
    nothing, and the next call runs normally."""
    import torch
    from linear_attention_ttt_b200 import synth
    from tests.gpu_util import upload_lact
    w = synth.make_lact(1, 2, 256, 128, 256, 64, synth.UPDATE_GD, seed=8)
    t = upload_lact(w)
    args = (t["q"], t["k"], t["v"], t["eta"], t["W1"], t["W2"], t["W3"], w.chunk)
    sentinel = torch.full((1, 2, 256, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    out = sentinel.clone()
    lib = ops.load()
    lib.ttt_test_fail_allocations(1)
    try:
        with pytest.raises(ops.TTTError) as e:
            ops.lact_swiglu_fwd(*args, out=out)
        assert e.value.code == -8   # TTT_ERR_ALLOC
    finally:
        lib.ttt_test_fail_allocations(0)
    torch.cuda.synchronize()
    assert torch.equal(out, sentinel)
    assert ops.device_status() == 0
    ref = ops.lact_swiglu_fwd(*args)
    again = ops.lact_swiglu_fwd(*args, out=out)
    torch.cuda.synchronize()
    assert torch.equal(ref, again)
    # the same hook reaches the other allocating entry points
    lib.ttt_test_fail_allocations(1)
    try:
        with pytest.raises(ops.TTTError) as e:
            ops.ttt_mlp_fwd(t["q"], t["k"], t["v"], t["eta"], t["W1"][:, :, :128],
                            torch.zeros(2, 256, device="cuda"), t["W2"][:, :, :256].contiguous(),
                            torch.zeros(2, 128, device="cuda"), 16)
        assert e.value.code == -8
    finally:
        lib.ttt_test_fail_allocations(0)
