"""Splitting one attention call over several GPUs by (batch, head).

Every (b, h) pair of an attention call is an independent problem: its output and
gradients depend on its own rows of Q, K, V and dO only.  So a call on (B, H, N, D)
tensors shards with no exchange at all: flatten (b, h) to bh = b*H + h, give each
of `world` ranks (or devices) a contiguous range of bh, run the library's kernels on
that range (a contiguous (1, count, N, D) view of the same memory), and, if every
rank needs the whole result, gather the ranges back.  The only collective is that
optional all-gather of outputs; the kernels themselves never communicate.

    head_ranges(B*H, world)                   contiguous, balanced bh ranges
    shard_view(t, rng)                         (1, count, N, D) view of t for a range
    sharded_attention(q, k, v, do, ...)        one rank's share, optionally all-gathered
    sharded_attention_devices(q, k, v, do, devices=...)   one process, several GPUs

The per-slice compute defaults to the library's CUDA entry points
(attention_forward / attention_backward); it is a parameter so that the partition
and reassembly logic can be tested on CPU ranks with a stand-in.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

from . import _binding


def head_ranges(bh: int, world: int) -> list[tuple[int, int]]:
    """Splits [0, bh) into `world` contiguous ranges whose sizes differ by at most one
    (the first bh % world ranges get the extra pair; ranges may be empty if world > bh)."""
    if bh < 0 or world < 1:
        raise ValueError(f"bad partition request: bh={bh}, world={world}")
    base, extra = divmod(bh, world)
    out, start = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((start, start + n))
        start += n
    return out


def shard_view(t: torch.Tensor | None, rng: tuple[int, int]):
    """The (1, count, N, D) (or (1, count, N) for lse) view of the pairs bh in rng of a
    contiguous (B, H, N, ...) tensor."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("sharding needs contiguous tensors")
    flat = t.reshape(t.shape[0] * t.shape[1], *t.shape[2:])
    return flat[rng[0]:rng[1]].unsqueeze(0)


def _cuda_compute(q, k, v, do, scale, causal):
    """One slice on its tensors' GPU through the library's C ABI."""
    o, lse = _binding.attention_forward(q, k, v, scale, causal)
    out = {"o": o, "lse": lse}
    if do is not None:
        out["dq"], out["dk"], out["dv"] = _binding.attention_backward(q, k, v, o, lse, do, scale, causal)
    return out


def _gather(local: torch.Tensor, ranges, rank: int, world: int, group, full_shape) -> torch.Tensor:
    """All-gathers each rank's (1, count, ...) slice into the full (B, H, ...) tensor (slices
    are padded to the largest range so that every rank sends the same number of bytes)."""
    dist = torch.distributed
    width = max(e - s for s, e in ranges)
    tail = local.shape[2:]
    send = torch.zeros((width, *tail), dtype=local.dtype, device=local.device)
    n = ranges[rank][1] - ranges[rank][0]
    if n:
        send[:n] = local[0]
    bufs = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(bufs, send, group=group)
    full = torch.empty((full_shape[0] * full_shape[1], *tail), dtype=local.dtype, device=local.device)
    for (s, e), b in zip(ranges, bufs):
        full[s:e] = b[: e - s]
    return full.view(*full_shape[:2], *tail)


def sharded_attention(q, k, v, do=None, scale: float | None = None, causal: bool = False, *, rank: int = 0,
                      world: int = 1, gather: bool = True, group=None,
                      compute: Callable | None = None):
    """This rank's share of attention (and, with do, its gradients) over (B, H, N, D)
    tensors that every rank holds in full.  Returns a dict with o, lse (and dq, dk, dv):
    the full tensors when `gather` (all-gathered over `group`), else this rank's
    (1, count, ...) slices plus the range itself under "range"."""
    B, H, N, D = q.shape
    scale = _binding.default_scale(D) if scale is None else scale
    compute = _cuda_compute if compute is None else compute
    ranges = head_ranges(B * H, world)
    rng = ranges[rank]
    res = compute(*(shard_view(t, rng) for t in (q, k, v, do)), scale, causal)
    if not gather:
        return {**res, "range": rng}
    if world == 1:
        return {n: t.view(B, H, *t.shape[2:]) for n, t in res.items()}
    return {n: _gather(t, ranges, rank, world, group, (B, H)) for n, t in res.items()}


def sharded_attention_devices(q, k, v, do=None, scale: float | None = None, causal: bool = False, *,
                              devices: Sequence[torch.device | int | str], compute: Callable | None = None):
    """One process, several GPUs: each device gets a contiguous range of (b, h) pairs (its
    slices are copied there), computes it on its own stream, and the results are copied
    back into full tensors on q's device.  No device waits on another's kernels."""
    B, H, N, D = q.shape
    scale = _binding.default_scale(D) if scale is None else scale
    compute = _cuda_compute if compute is None else compute
    devs = [torch.device(d) if not isinstance(d, int) else torch.device("cuda", d) for d in devices]
    ranges = head_ranges(B * H, len(devs))
    parts = []
    for dev, rng in zip(devs, ranges):
        if rng[0] == rng[1]:
            continue
        with torch.cuda.device(dev) if dev.type == "cuda" else _nullctx():
            ins = [None if t is None else shard_view(t, rng).to(dev, non_blocking=True) for t in (q, k, v, do)]
            parts.append((rng, compute(*ins, scale, causal)))
    out = {}
    for rng, res in parts:
        for n, t in res.items():
            if n not in out:
                out[n] = torch.empty((B * H, *t.shape[2:]), dtype=t.dtype, device=q.device)
            out[n][rng[0]:rng[1]] = t[0].to(q.device)
    return {n: t.view(B, H, *t.shape[1:]) for n, t in out.items()}


class _nullctx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False
