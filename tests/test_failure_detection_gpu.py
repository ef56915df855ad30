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
