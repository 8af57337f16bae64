"""Head partition of the PR-Sink step over several GPUs (one process per GPU).

The pages run the 14B DiT on 2 (or 4) GPUs with Ulysses sequence parallelism, whose
all-to-all gives every GPU all tokens of a subset of the attention heads (LiveAnimate digest,
pipeline paragraph, last sentence; news article, "three key breakthroughs", item 3).  Heads are
independent in every step of this path: attention, the KV append, the dynamic-sink fill and
the bank store each touch one head's rows at a time.  So rank r of N holds heads
[h0, h1) = head_range(H, N, r) of every cache and bank entry and runs the same calls with a
layout whose ``n_heads`` is h1 - h0; no collective is needed inside the path.  The pose side
(fingerprint, retrieval decision, bank decision) is 11 KB of deterministic work on the same
inputs, so every rank computes it itself and all ranks take identical decisions.

These helpers only slice and reassemble host- or device-side tensors; they hold none of the
method's arithmetic.
"""
from __future__ import annotations

import torch


def head_range(n_heads: int, world: int, rank: int):
    """Contiguous heads of ``rank``: [h0, h1).  Sizes differ by at most one head when
    ``n_heads`` is not a multiple of ``world``; every rank gets at least one head."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n_heads < world:
        raise ValueError(f"{n_heads} heads cannot be split over {world} ranks")
    base, extra = divmod(n_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_config(cfg: dict, world: int, rank: int) -> dict:
    """The layout fields of ``rank``'s shard: the same geometry with its head count."""
    h0, h1 = head_range(int(cfg["n_heads"]), world, rank)
    return dict(cfg, n_heads=h1 - h0)


def shard_tokens(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """Rank's heads of a token-major tensor ``[L][H][d]`` (q, k_new, v_new, out), contiguous."""
    h0, h1 = head_range(x.shape[1], world, rank)
    return x[:, h0:h1].contiguous()


def shard_heads(x: torch.Tensor, world: int, rank: int, axis: int) -> torch.Tensor:
    """Rank's heads of a tensor whose head axis is ``axis`` (caches ``[..][H][T][d]``, bank
    entries ``[..][H][L_blk][d]``, LSE ``[H][L_blk]``), contiguous."""
    h0, h1 = head_range(x.shape[axis], world, rank)
    return x.narrow(axis, h0, h1 - h0).contiguous()


def gather_heads(parts, axis: int) -> torch.Tensor:
    """Reassemble the per-rank shards (in rank order) along the head axis."""
    return torch.cat(list(parts), dim=axis)
