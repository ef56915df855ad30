"""Seeded synthetic inputs for the chunked TTT-layer forward pass.

This module only draws and rounds numbers; it holds none of the method's
arithmetic. It is the one piece shared by the CUDA path's tests/bench and the
CPU oracle: both receive the same arrays from here.

Recipe (per workload): ``numpy.random.Generator(PCG64(seed))``; draw order
q, k, v, eta-noise, then the fast-weight initialisation. Values are drawn in
float64, optionally L2-normalised per token in float64, then rounded
(float64 -> float32 round-to-nearest-even, then float32 -> bfloat16
round-to-nearest-even for bf16 workloads). The arrays returned are float32
holding exactly the stored values, so uploading them as bf16 is exact and the
oracle's float64 upcast is exact.

Workload shapes follow the pages' settings: the TTT layer of the
"Test-Time Training (TTT)" summary (head dim 64, chunk 16..256, per-token
learning rate eta = sigmoid(.) or a small softplus), and LaCT's large-chunk
SwiGLU fast weights ("Test-Time Training Done Right" review, sections 2-4:
chunks of 2K+ tokens, 32K-token training length).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"

LOSS_MSE = 0
LOSS_NEG_DOT = 1
UPDATE_GD = 0
UPDATE_MUON = 1


def round_to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (RNE from the float32 value), returned as float32."""
    f = round_to_f32(x)
    u = f.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    u = ((u + bias) & np.uint64(0xFFFF0000)).astype(np.uint32)
    return u.view(np.float32)


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are exactly bf16-representable."""
    return (np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _l2n(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 0.5 * (1.0 + np.tanh(0.5 * x))


@dataclass
class Workload:
    name: str
    variant: str            # "ttt_linear" or "lact"
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: str              # F32 or BF16: storage type of q, k, v and out
    loss: int = LOSS_MSE    # ttt_linear only
    dh: int = 0             # lact only
    update_rule: int = UPDATE_GD
    causal: int = 1
    seed: int = 0
    q: Optional[np.ndarray] = None
    k: Optional[np.ndarray] = None
    v: Optional[np.ndarray] = None
    eta: Optional[np.ndarray] = None
    W0: Optional[np.ndarray] = None     # ttt_linear: [H,dk,dv] or [B,H,dk,dv]
    W1: Optional[np.ndarray] = None     # lact: [H,dh,dk]
    W2: Optional[np.ndarray] = None     # lact: [H,dv,dh]
    W3: Optional[np.ndarray] = None     # lact: [H,dh,dk]
    meta: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def f64(self, name: str) -> np.ndarray:
        return np.asarray(getattr(self, name), dtype=np.float64)


def _draw_tokens(rng, shape, scale, normalise, dtype):
    x = rng.standard_normal(shape)
    if normalise:
        x = _l2n(x)
    x = x * scale
    return round_to_bf16(x) if dtype == BF16 else round_to_f32(x)


def make_ttt_linear(B, H, T, dk, dv, chunk, dtype, loss, seed, *, qk_norm=True,
                    v_norm=False, token_scale=1.0, eta_kind="const", eta_scale=0.1,
                    w0_std=0.02, w0_batched=False, name="custom") -> Workload:
    """TTT-Linear / inner-product workload. eta_kind: const | sigmoid | softplus."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _draw_tokens(rng, (B, H, T, dk), token_scale, qk_norm, dtype)
    k = _draw_tokens(rng, (B, H, T, dk), token_scale, qk_norm, dtype)
    v = _draw_tokens(rng, (B, H, T, dv), token_scale, v_norm, dtype)
    noise = rng.standard_normal((B, H, T))
    if eta_kind == "const":
        eta = np.full((B, H, T), eta_scale)
    elif eta_kind == "sigmoid":
        eta = eta_scale * _sigmoid(noise)
    elif eta_kind == "softplus":
        eta = eta_scale * _softplus(noise)
    else:
        raise ValueError(eta_kind)
    wshape = (B, H, dk, dv) if w0_batched else (H, dk, dv)
    W0 = rng.standard_normal(wshape) * w0_std if w0_std > 0 else np.zeros(wshape)
    return Workload(name=name, variant="ttt_linear", B=B, H=H, T=T, dk=dk, dv=dv,
                    chunk=chunk, dtype=dtype, loss=loss, seed=seed, q=q, k=k, v=v,
                    eta=round_to_f32(eta), W0=round_to_f32(W0))


def make_lact(B, H, T, d, dh, chunk, update_rule, seed, *, causal=1, dtype=BF16,
              eta_scale=1e-3, name="custom") -> Workload:
    """LaCT SwiGLU workload: L2-normalised q, k, v; W ~ N(0, 1/fan_in) per head."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _draw_tokens(rng, (B, H, T, d), 1.0, True, dtype)
    k = _draw_tokens(rng, (B, H, T, d), 1.0, True, dtype)
    v = _draw_tokens(rng, (B, H, T, d), 1.0, True, dtype)
    eta = eta_scale * _softplus(rng.standard_normal((B, H, T)))
    W1 = rng.standard_normal((H, dh, d)) / np.sqrt(d)
    W3 = rng.standard_normal((H, dh, d)) / np.sqrt(d)
    W2 = rng.standard_normal((H, d, dh)) / np.sqrt(dh)
    return Workload(name=name, variant="lact", B=B, H=H, T=T, dk=d, dv=d, dh=dh,
                    chunk=chunk, dtype=dtype, update_rule=update_rule, causal=causal,
                    seed=seed, q=q, k=k, v=v, eta=round_to_f32(eta),
                    W1=round_to_f32(W1), W2=round_to_f32(W2), W3=round_to_f32(W3))


# The five named workloads. Sizes, value distributions and seeds are fixed here.
CONFIG_NAMES = {
    1: "ttt_linear_mse_f32_B1_H2_T256_d64_b16",
    2: "linear_attention_bf16_B4_H16_T4096_d128_b64",
    3: "ttt_linear_mse_bf16_B8_H16_T8192_d64",
    4: "lact_swiglu_gd_B2_H4_T32768_d256_dh512_b2048",
    5: "lact_swiglu_muon_B1_H8_T131072_d128_dh512_b4096",
}


def config(index: int, chunk: Optional[int] = None, T: Optional[int] = None,
           B: Optional[int] = None, H: Optional[int] = None, replica: int = 0) -> Workload:
    """Named workload ``index`` (1..5); T/B/H overrides give smaller cases with
    the same distributions (used for parity runs the oracle finishes quickly).
    ``replica`` > 0 draws an independent batch of the same workload (one per
    rank of a multi-GPU run)."""
    seed = 1000 + index + 100 * replica
    if index == 1:
        w = make_ttt_linear(B or 1, H or 2, T or 256, 64, 64, chunk or 16, F32, LOSS_MSE,
                            seed, qk_norm=True, eta_kind="const", eta_scale=0.1, w0_std=0.02)
    elif index == 2:
        w = make_ttt_linear(B or 4, H or 16, T or 4096, 128, 128, chunk or 64, BF16,
                            LOSS_NEG_DOT, seed, qk_norm=False, token_scale=1.0 / np.sqrt(128),
                            eta_kind="sigmoid", eta_scale=0.1, w0_std=0.0)
    elif index == 3:
        w = make_ttt_linear(B or 8, H or 16, T or 8192, 64, 64, chunk or 16, BF16, LOSS_MSE,
                            seed, qk_norm=True, eta_kind="softplus", eta_scale=0.05,
                            w0_std=0.02)
    elif index == 4:
        w = make_lact(B or 2, H or 4, T or 32768, 256, 512, chunk or 2048, UPDATE_GD, seed)
    elif index == 5:
        w = make_lact(B or 1, H or 8, T or 131072, 128, 512, chunk or 4096, UPDATE_MUON, seed)
    else:
        raise ValueError(f"no workload {index}")
    w.name = (CONFIG_NAMES[index] + ("" if chunk is None else f"_chunk{chunk}") +
              ("" if T is None else f"_T{T}"))
    w.meta["config"] = index
    return w
