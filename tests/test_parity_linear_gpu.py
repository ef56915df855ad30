"""GPU parity of ttt_linear_fwd (C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import ops, synth
from tests.gpu_util import check, run_linear, upload_linear, max_row_rel

pytestmark = pytest.mark.gpu


def oracle_linear(w, definition=False):
    fn = O.ttt_linear_minibatch if definition else O.ttt_linear_dual
    return fn(w.q, w.k, w.v, w.eta, w.W0, w.chunk, w.loss)


def test_f32_mse_full_size_workload():
    """TTT-Linear MSE, fp32, batch 1, 2 heads, T=256, d=64, chunk 16."""
    w = synth.config(1)
    y, Wf = run_linear(w)
    yo, Wo = oracle_linear(w, definition=True)
    check(y, yo, w.dtype, "y")
    check(Wf, Wo, w.dtype, "W_final")


@pytest.mark.parametrize("loss", [ops.TTT_LOSS_MSE, ops.TTT_LOSS_NEG_DOT])
@pytest.mark.parametrize("T,chunk", [(1, 16), (37, 16), (40, 1), (33, 64), (100, 7), (64, 64)])
def test_f32_ragged_and_degenerate_chunks(loss, T, chunk):
    w = synth.make_ttt_linear(2, 2, T, 64, 64, chunk, synth.F32, loss, seed=T * 7 + chunk,
                              eta_kind="softplus", eta_scale=0.05)
    y, Wf = run_linear(w)
    yo, Wo = oracle_linear(w, definition=True)
    check(y, yo, w.dtype, "y")
    check(Wf, Wo, w.dtype, "W_final")


@pytest.mark.parametrize("dk,dv", [(16, 16), (48, 80), (128, 128), (256, 256), (256, 40)])
def test_f32_head_sizes(dk, dv):
    w = synth.make_ttt_linear(1, 2, 45, dk, dv, 16, synth.F32, ops.TTT_LOSS_MSE, seed=dk + dv,
                              eta_kind="softplus", eta_scale=0.05)
    y, Wf = run_linear(w)
    yo, Wo = oracle_linear(w)
    check(y, yo, w.dtype, "y")
    check(Wf, Wo, w.dtype, "W_final")


def test_f32_per_sequence_w0_and_strided_tokens():
    """W0 given per (batch, head), and q/k/v/out as [B,T,H,d] storage viewed
    as [B,H,T,d] (non-contiguous strides)."""
    w = synth.make_ttt_linear(3, 4, 50, 64, 64, 16, synth.F32, ops.TTT_LOSS_MSE, seed=5,
                              eta_kind="sigmoid", eta_scale=0.1, w0_batched=True)
    t = upload_linear(w)
    for n in ("q", "k", "v"):
        t[n] = t[n].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    out = torch.empty((3, 50, 4, 64), device="cuda").permute(0, 2, 1, 3)
    ops.ttt_linear_fwd(t["q"], t["k"], t["v"], t["eta"], t["W0"], 16, ops.TTT_LOSS_MSE, out=out)
    torch.cuda.synchronize()
    yo, _ = oracle_linear(w)
    check(out.cpu().numpy(), yo, w.dtype, "y")


def test_f32_empty_sequence_copies_w0():
    w = synth.make_ttt_linear(2, 2, 0, 64, 64, 16, synth.F32, ops.TTT_LOSS_MSE, seed=1)
    y, Wf = run_linear(w)
    assert y.shape == (2, 2, 0, 64)
    assert np.array_equal(Wf, np.broadcast_to(w.W0, Wf.shape))


def test_f32_zero_learning_rate():
    w = synth.make_ttt_linear(1, 2, 40, 64, 64, 16, synth.F32, ops.TTT_LOSS_MSE, seed=2)
    w.eta[:] = 0
    y, Wf = run_linear(w)
    assert np.array_equal(Wf, np.broadcast_to(w.W0, Wf.shape))
    assert max_row_rel(y, np.einsum("bhta,hac->bhtc", w.q.astype(np.float64), w.W0)) < 1e-5


def test_f32_resume_from_w_final():
    w = synth.make_ttt_linear(2, 2, 96, 64, 64, 16, synth.F32, ops.TTT_LOSS_MSE, seed=3,
                              eta_kind="softplus", eta_scale=0.05)
    t = upload_linear(w)
    y, Wf = ops.ttt_linear_fwd(t["q"], t["k"], t["v"], t["eta"], t["W0"], 16, 0)
    ya, Wa = ops.ttt_linear_fwd(t["q"][:, :, :48], t["k"][:, :, :48], t["v"][:, :, :48],
                                t["eta"][:, :, :48], t["W0"], 16, 0)
    yb, Wb = ops.ttt_linear_fwd(t["q"][:, :, 48:], t["k"][:, :, 48:], t["v"][:, :, 48:],
                                t["eta"][:, :, 48:].contiguous(), Wa, 16, 0)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([ya, yb], dim=2), y)
    assert torch.equal(Wb, Wf)


# ---------------------------------------------------------------------------
# bf16 tokens, fp32 state
# ---------------------------------------------------------------------------

def test_bf16_linear_attention_full_size_workload():
    """Inner-product loss (chunked causal linear attention): batch 4, 16
    heads, T=4096, d=128, chunk 64, bf16, W0=0, eta=0.1*sigmoid(N(0,1))."""
    w = synth.config(2)
    y, Wf = run_linear(w)
    yo, Wo = oracle_linear(w)
    check(y, yo, w.dtype, "y")
    check(Wf, Wo, w.dtype, "W_final")


@pytest.mark.parametrize("chunk", [16, 256])
def test_bf16_mse_full_size_workload(chunk):
    """TTT-Linear MSE: batch 8, 16 heads, T=8192, d=64, bf16, chunk 16/256."""
    w = synth.config(3, chunk=chunk)
    y, Wf = run_linear(w)
    yo, Wo = oracle_linear(w)
    check(y, yo, w.dtype, "y")
    check(Wf, Wo, w.dtype, "W_final")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("loss", [ops.TTT_LOSS_MSE, ops.TTT_LOSS_NEG_DOT])
@pytest.mark.parametrize("T,chunk", [(1, 16), (37, 16), (300, 64), (100, 5), (70, 24), (64, 256),
                                     (200, 32), (130, 128)])
def test_bf16_ragged_and_odd_chunks(d, loss, T, chunk):
    w = synth.make_ttt_linear(2, 3, T, d, d, chunk, synth.BF16, loss, seed=T + chunk + d,
                              eta_kind="softplus", eta_scale=0.05)
    y, Wf = run_linear(w)
    yo, Wo = oracle_linear(w, definition=True)
    check(y, yo, w.dtype, "y")
    check(Wf, Wo, w.dtype, "W_final")


def test_bf16_per_sequence_w0_strided_tokens_and_empty():
    w = synth.make_ttt_linear(2, 3, 80, 64, 64, 16, synth.BF16, ops.TTT_LOSS_MSE, seed=11,
                              eta_kind="softplus", eta_scale=0.05, w0_batched=True)
    t = upload_linear(w)
    for n in ("q", "k", "v"):
        t[n] = t[n].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    out = torch.empty((2, 80, 3, 64), device="cuda", dtype=torch.bfloat16).permute(0, 2, 1, 3)
    _, Wf = ops.ttt_linear_fwd(t["q"], t["k"], t["v"], t["eta"], t["W0"], 16, 0, out=out)
    torch.cuda.synchronize()
    yo, Wo = oracle_linear(w)
    check(out.float().cpu().numpy(), yo, w.dtype, "y")
    check(Wf.cpu().numpy(), Wo, w.dtype, "W_final")
    e = synth.make_ttt_linear(1, 2, 0, 128, 128, 64, synth.BF16, ops.TTT_LOSS_NEG_DOT, seed=1)
    y, Wf = run_linear(e)
    assert np.array_equal(Wf, np.broadcast_to(e.W0, Wf.shape))


@pytest.mark.parametrize("loss", [ops.TTT_LOSS_MSE, ops.TTT_LOSS_NEG_DOT])
@pytest.mark.parametrize("split", [128, 96])
def test_bf16_resume_from_w_final(loss, split):
    """Running a prefix, then the rest from its W_final, equals one run. The
    d = 64 MSE kernel works in 64-token groups: a split on a group boundary is
    bit-exact; any other chunk-aligned split differs only by rounding order."""
    w = synth.make_ttt_linear(2, 2, 256, 64, 64, 32, synth.BF16, loss, seed=4,
                              eta_kind="softplus", eta_scale=0.05)
    t = upload_linear(w)
    y, Wf = ops.ttt_linear_fwd(t["q"], t["k"], t["v"], t["eta"], t["W0"], 32, loss)
    sl = lambda x, a, b: x[:, :, a:b]
    ya, Wa = ops.ttt_linear_fwd(sl(t["q"], 0, split), sl(t["k"], 0, split), sl(t["v"], 0, split),
                                sl(t["eta"], 0, split), t["W0"], 32, loss)
    yb, Wb = ops.ttt_linear_fwd(sl(t["q"], split, 256), sl(t["k"], split, 256),
                                sl(t["v"], split, 256), sl(t["eta"], split, 256), Wa, 32, loss)
    torch.cuda.synchronize()
    yc = torch.cat([ya, yb], dim=2)
    if split % 64 == 0:
        assert torch.equal(yc, y)
        assert torch.equal(Wb, Wf)
    else:
        yo, Wo = oracle_linear(w)
        check(yc.float().cpu().numpy(), yo, synth.BF16, "resumed y")
        check(Wb.float().cpu().numpy(), Wo, synth.BF16, "resumed W_final")


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (48, 48), (80, 80), (256, 256),
                                   (64, 32), (32, 128), (128, 48)])
@pytest.mark.parametrize("loss", [ops.TTT_LOSS_MSE, ops.TTT_LOSS_NEG_DOT])
def test_bf16_other_head_sizes(dk, dv, loss):
    """bf16 head sizes without a tensor-core kernel (any multiple of 16 up to
    256, dk != dv) run the CUDA-core kernel; ragged last chunk."""
    w = synth.make_ttt_linear(2, 2, 70, dk, dv, 16, synth.BF16, loss, seed=dk + 3 * dv,
                              eta_kind="softplus", eta_scale=0.05)
    y, Wf = run_linear(w)
    yo, Wo = oracle_linear(w, definition=True)
    check(y, yo, w.dtype, f"y dk{dk} dv{dv}")
    check(Wf, Wo, w.dtype, f"W_final dk{dk} dv{dv}")


def test_oversized_head_is_rejected():
    w = synth.make_ttt_linear(1, 1, 16, 32, 32, 16, synth.BF16, 0, seed=1)
    t = upload_linear(w)
    q = torch.zeros((1, 1, 16, 272), dtype=torch.bfloat16, device="cuda")
    W0 = torch.zeros((1, 272, 32), device="cuda")
    with pytest.raises(ops.TTTError) as e:
        ops.ttt_linear_fwd(q, q, t["v"], t["eta"], W0, 16, 0)
    assert e.value.code == -5
