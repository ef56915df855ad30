"""Context-parallel LaCT: the tokens of every large chunk split over ranks
("Test-Time Training Done Right" review, section 8: each device computes the
update gradient of its share of a chunk and the shares are summed).

Rank r of R holds sub-block r (chunk/R tokens) of every chunk. The layer
runs as one ``lact_swiglu_fwd_cp`` call per rank; the library calls back once
per chunk with its fp32 gradient buffer, and the callback sums it over the
ranks with ``torch.distributed.all_reduce`` (NCCL on GPUs) on the layer's
stream. Newton-Schulz, the step and the renorm then run on identical data on
every rank, so the fast weights stay identical everywhere.

This module is argument marshalling and plumbing: the shard layout, the
callback that wraps the library's buffer as a tensor for the collective, and
the call itself.
"""
from __future__ import annotations

import ctypes

import torch

from . import ops

REDUCE_FN = ops.REDUCE_FN


def shard(x: torch.Tensor, rank: int, world: int, chunk: int) -> torch.Tensor:
    """Rank `rank`'s tokens of x [B,H,T,...] (T a multiple of chunk, chunk a
    multiple of world): sub-block `rank` of every chunk, in order."""
    B, H, T = x.shape[:3]
    if T % chunk or chunk % world:
        raise ValueError("T must be a multiple of chunk and chunk a multiple of world")
    cl = chunk // world
    v = x.reshape(B, H, T // chunk, world, cl, *x.shape[3:])
    return v[:, :, :, rank].reshape(B, H, T // world, *x.shape[3:]).contiguous()


def unshard(parts, chunk: int) -> torch.Tensor:
    """Inverse of ``shard``: the ranks' pieces back in token order."""
    world = len(parts)
    B, H, Tl = parts[0].shape[:3]
    cl = chunk // world
    st = torch.stack([p.reshape(B, H, Tl // cl, cl, *p.shape[3:]) for p in parts], dim=3)
    return st.reshape(B, H, Tl * world, *parts[0].shape[3:])


class _CudaBuffer:
    """A device buffer described by __cuda_array_interface__, so that torch
    can alias it without copying."""

    def __init__(self, ptr: int, n: int, stream: int):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (ptr, False),
                                         "version": 3, "stream": stream or None}


def make_reducer(reduce_tensor):
    """Wraps `reduce_tensor(t)` (an in-place sum of a CUDA fp32 tensor over
    the ranks, enqueued on torch's current stream) as the library's
    callback. Returns the ctypes function (keep a reference while the call
    runs)."""

    def cb(ptr, n, stream, _user):
        try:
            s = torch.cuda.ExternalStream(stream) if stream else torch.cuda.default_stream()
            with torch.cuda.stream(s):
                t = torch.as_tensor(_CudaBuffer(ptr, n, stream or 0), device="cuda")
                reduce_tensor(t)
            return 0
        except Exception:  # reported to the library as a failed exchange
            return 1

    return REDUCE_FN(cb)


def dist_reducer(group=None):
    """Gradient exchange over a torch.distributed process group."""
    import torch.distributed as dist
    return make_reducer(lambda t: dist.all_reduce(t, group=group))


def lact_swiglu_fwd_cp(q, k, v, eta, W1, W2, W3, chunk_local: int, update_rule: int, reducer,
                       causal: int = 1, out=None, finals=False, stream=None):
    """One rank's share of the context-parallel LaCT layer. q, k, v, eta are
    this rank's shards (``shard``); chunk_local = chunk / world; `reducer`
    comes from ``dist_reducer`` or ``make_reducer`` (None: one rank)."""
    B, H, T, dk = q.shape
    dv, dh = v.shape[-1], W1.shape[-2]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    F = [None, None, None]
    if finals:
        F = [torch.empty(s, dtype=torch.float32, device=q.device)
             for s in ((B, H, dh, dk), (B, H, dv, dh), (B, H, dh, dk))]
    ds = [ops.describe(x) for x in (q, k, v, eta, W1, W2, W3, out, *F)]
    r = [ops._ref(d) for d in ds]
    fn = reducer if reducer is not None else ctypes.cast(None, REDUCE_FN)
    code = ops.load().lact_swiglu_fwd_cp(*r[:7], int(chunk_local), int(update_rule), int(causal),
                                         r[7], r[8], r[9], r[10], fn, None, ops._stream(stream))
    ops._check(code, "lact_swiglu_fwd_cp")
    return (out, *F) if finals else out
