"""Sequence sharding of the mixer's attention cores over ranks, one GPU each.

A long video's tokens are split into contiguous shards, one per rank. The
per-token parts of a layer (the projections, the router, the gates) need
nothing from other ranks; the two attention cores do:

* gated linear attention: its state is a sum over tokens, so each rank forms
  the state of its own shard (sva_linear_attn_state_fwd), one all-reduce sums
  the states (fp32, B*H*(d*d + d) values: 1.58 MB per 720p layer), and each
  rank reads out its own queries (sva_linear_attn_readout_fwd);
* the gated softmax anchor: every query sees every key, so each rank
  all-gathers K and V (2*N*D values) and runs the anchor for its own queries
  against all keys (sva_softmax_anchor_fwd with n_keys = N).

The collectives go through torch.distributed (NCCL between GPUs, over NVLink
on one node); every step of the attention itself runs in the library's
kernels. `ops` replaces those kernel calls (used by host-logic tests that run
on CPU ranks); by default they are the library's entry points.
"""
from __future__ import annotations

from types import SimpleNamespace
from typing import List, Optional, Tuple


def shard_bounds(n_tokens: int, world: int, rank: int) -> Tuple[int, int]:
    """[start, stop) of rank's contiguous token shard; the first n_tokens % world
    ranks hold one token more."""
    if world < 1 or not 0 <= rank < world or n_tokens < world:
        raise ValueError(f"cannot shard {n_tokens} tokens over {world} ranks (rank {rank})")
    base, extra = divmod(n_tokens, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_lengths(n_tokens: int, world: int) -> List[int]:
    return [b - a for a, b in (shard_bounds(n_tokens, world, r) for r in range(world))]


def library_ops():
    """The library's kernels as the compute steps of the sharded cores."""
    from . import (sva_linear_attn_readout_fwd, sva_linear_attn_state_bytes,
                   sva_linear_attn_state_fwd, sva_softmax_anchor_fwd)
    return SimpleNamespace(state_bytes=sva_linear_attn_state_bytes,
                           state_fwd=sva_linear_attn_state_fwd,
                           readout_fwd=sva_linear_attn_readout_fwd,
                           anchor_fwd=sva_softmax_anchor_fwd)


def _dist():
    import torch.distributed as dist
    if not dist.is_initialized():
        raise RuntimeError("torch.distributed is not initialised")
    return dist


def sharded_linear_attn(q, k, v, gate, out, H: int, group=None, eps: float = 1e-6,
                        flags: int = 0, wgate=None, residual=None, ops=None):
    """Gated linear attention of this rank's token shard against the state of
    the whole sequence. q, k, v, gate, out (residual, wgate) hold this rank's
    tokens [B, n_local, ...]. Returns the summed state (fp32)."""
    import torch
    ops = ops or library_ops()
    B, _, D = k.shape
    d = D // H
    state = torch.empty(ops.state_bytes(B, H, d) // 4, dtype=torch.float32, device=k.device)
    ops.state_fwd(k, v, state, H, flags=flags, wgate=wgate)
    _dist().all_reduce(state, group=group)
    ops.readout_fwd(q, gate, out, state, H, residual=residual, eps=eps, flags=flags)
    return state


def gather_tokens(x, n_tokens: int, group=None):
    """All-gather the contiguous token shards [B, n_r, W] of every rank into the
    whole sequence [B, n_tokens, W] (ragged shards are padded for the
    collective and trimmed after)."""
    import torch
    dist = _dist()
    world = dist.get_world_size(group)
    lens = shard_lengths(n_tokens, world)
    B, n, W = x.shape
    if n != lens[dist.get_rank(group)]:
        raise ValueError(f"this rank holds {n} tokens, its shard has {lens[dist.get_rank(group)]}")
    m = max(lens)
    pad = torch.zeros(B, m, W, dtype=x.dtype, device=x.device)
    pad[:, :n] = x
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :l] for p, l in zip(parts, lens)], dim=1).contiguous()


def sharded_anchor(q, k, v, gate, out, H: int, n_tokens: int, group=None, scale: float = 0.0,
                   residual=None, ops=None):
    """Gated softmax anchor of this rank's queries against all n_tokens keys:
    K and V are all-gathered, then the anchor runs with n_keys = n_tokens."""
    ops = ops or library_ops()
    K = gather_tokens(k, n_tokens, group)
    V = gather_tokens(v, n_tokens, group)
    ops.anchor_fwd(q, K, V, gate, out, H, residual=residual, scale=scale)
    return K, V
