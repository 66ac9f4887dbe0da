"""Splitting one problem of the path over ranks (one process per GPU).

The path's independent units are (batch, kv head) pairs: a kv head's group of
query heads is scored against that kv head's pooled keys alone, and each query
tile's attention reads only its own kv head's tiles. Per-head scoring
therefore splits over units with no collective on the data path: a rank runs
the whole path on its units' heads.

Head-shared scoring is the exception: the keep is computed once from the
means over all heads of the pooled q and k (selector.py, score_blocks with
head_shared), so every rank needs every head's pooled vectors. The exchange is
one all-gather of the pooled vectors (B, heads of the rank, NQ, D) and
(B, kv heads of the rank, NK, D), float32, a few MB at the workloads' sizes;
every rank then runs the same selection on the gathered tensors, so all
ranks hold the same keep as a single GPU would compute from those inputs.

This module holds the partition and the exchange only; the arithmetic runs in
the library's kernels on each rank.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Box:
    """A rectangle of units: batches [b0, b1) x kv heads [hk0, hk1). Its q
    slice is q[b0:b1, hk0*g:hk1*g] and its k, v slices k[b0:b1, hk0:hk1]; a
    box either lies in one batch or covers every kv head of its batches, so
    each slice is contiguous in the (B, H, S, D) layout."""
    b0: int
    b1: int
    hk0: int
    hk1: int

    def units(self):
        return [(b, hk) for b in range(self.b0, self.b1) for hk in range(self.hk0, self.hk1)]


def units(B: int, Hkv: int):
    """Every (batch, kv head) unit, batch-major."""
    return [(b, hk) for b in range(B) for hk in range(Hkv)]


def rank_range(n: int, rank: int, world: int):
    """The contiguous, balanced share [lo, hi) of n items that `rank` owns."""
    if not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside world {world}")
    return n * rank // world, n * (rank + 1) // world


def rank_boxes(B: int, Hkv: int, rank: int, world: int):
    """The rank's units (a contiguous run of the batch-major unit list) as at
    most three boxes: the tail of a first batch, whole batches, the head of
    a last batch. Every unit belongs to exactly one rank."""
    lo, hi = rank_range(B * Hkv, rank, world)
    boxes = []
    u = lo
    while u < hi:
        b, hk = divmod(u, Hkv)
        if hk == 0 and hi - u >= Hkv:
            nb = (hi - u) // Hkv  # whole batches
            boxes.append(Box(b, b + nb, 0, Hkv))
            u += nb * Hkv
        else:
            end = min(hi - b * Hkv, Hkv)  # within batch b
            boxes.append(Box(b, b + 1, hk, end))
            u = b * Hkv + end
    return boxes


def gather_heads(local: torch.Tensor, counts, group=None) -> torch.Tensor:
    """All-gather along the head axis (dim 1) of per-rank blocks of pooled
    vectors: rank r contributes `local` with counts[r] heads (its boxes'
    heads, in unit order); returns the (B, sum(counts), N, D) tensor in rank
    order, i.e. in head order when every rank's heads are one contiguous
    range. Uneven counts are padded for the collective and cut after it."""
    world = len(counts)
    width = max(counts)
    B, _, N, D = local.shape
    pad = local.new_zeros(B, width, N, D)
    pad[:, :local.shape[1]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    torch.distributed.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, :c] for p, c in zip(parts, counts)], dim=1)


def head_range(Hkv: int, rank: int, world: int):
    """The contiguous kv heads [lo, hi) that `rank` owns when the heads of
    every batch are split (head-shared scoring, B = 1 or every batch split
    the same way)."""
    return rank_range(Hkv, rank, world)
