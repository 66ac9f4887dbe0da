"""Oracle for the selection half of the path: pool, score, plan, top-k keep.

TEST INFRASTRUCTURE ONLY (see the package docstring). Follows the functions of
the page "automatic/modules/attention/sparse/selector.py" in their order and
notation; each function names the one it restates. Arrays are NumPy; floating
point is float64 unless stated.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class SparseSpec:
    """selector.py, ``SparseSpec``: budget is a fraction of the candidates
    (tiles neither forced nor forbidden); pinned and diagonal tiles come on
    top of it. ``score_chunk_bytes`` only bounds memory in the page's scorer
    and does not change any result, so it is not carried here."""
    budget: float = 0.30
    block_q: int = 128
    block_kv: int = 64
    head_shared: bool = False
    force: bool = False


def block_count(length: int, block: int) -> int:
    """selector.py, ``block_count``: ceil(length / block)."""
    return (length + block - 1) // block


def pool_blocks(x: np.ndarray, block: int) -> np.ndarray:
    """selector.py, ``pool_blocks``: mean of each run of ``block`` tokens.

    ``x`` has tokens on axis -2. Tile i covers tokens [i*block,
    min((i+1)*block, S)); a partial final tile is averaged over its own token
    count, not over ``block``. The sum is float64 (exact for bf16 inputs at
    these lengths) followed by one division.
    """
    x = np.asarray(x, dtype=np.float64)
    S = x.shape[-2]
    n = block_count(S, block)
    out = np.empty(x.shape[:-2] + (n, x.shape[-1]), dtype=np.float64)
    for i in range(n):
        lo, hi = i * block, min((i + 1) * block, S)
        out[..., i, :] = x[..., lo:hi, :].sum(axis=-2) / float(hi - lo)
    return out


def diagonal_blocks(nq: int, nk: int, block_q: int, block_kv: int) -> np.ndarray:
    """selector.py, ``diagonal_blocks``: tile (i, j) is diagonal when the
    nominal token ranges [i*bq, (i+1)*bq) and [j*bkv, (j+1)*bkv) overlap.
    Raw token indices: no clamp to the sequence lengths and no rescaling when
    the query and key lengths differ."""
    i = np.arange(nq, dtype=np.int64)[:, None]
    j = np.arange(nk, dtype=np.int64)[None, :]
    return (i * block_q < (j + 1) * block_kv) & (j * block_kv < (i + 1) * block_q)


def head_map(pq: np.ndarray, pk: np.ndarray, head_shared: bool):
    """selector.py, ``score_blocks`` head handling.

    head_shared: both pooled tensors are averaged over their head axis, giving
    one keep head. Otherwise, when the key has fewer heads (GQA), query head h
    is paired with key head h // (Hq / Hkv) (repeat-interleave).
    """
    Hq, Hkv = pq.shape[1], pk.shape[1]
    if head_shared:
        return pq.mean(axis=1, keepdims=True), pk.mean(axis=1, keepdims=True)
    if Hkv != Hq:
        if Hq % Hkv:
            raise ValueError("query heads must be a multiple of key heads")
        pk = np.repeat(pk, Hq // Hkv, axis=1)
    return pq, pk


def score_blocks(q: np.ndarray, k: np.ndarray, spec: SparseSpec) -> np.ndarray:
    """selector.py, ``score_blocks``: unscaled pooled affinity per tile pair,
    S[b, h, i, j] = <pooled_q[b, h, i], pooled_k[b, h', j]>. No softmax scale
    and no softmax: neither changes the top-k order. Returns (B, Hs, NQ, NK)."""
    pq = pool_blocks(q, spec.block_q)
    pk = pool_blocks(k, spec.block_kv)
    pq, pk = head_map(pq, pk, spec.head_shared)
    return np.matmul(pq, np.swapaxes(pk, -1, -2))


def budget_count(per_row, budget: float) -> np.ndarray:
    """Tiles a row may choose: ceil(per_row * budget).

    In selection_plan the product is an int64 tensor times a Python float,
    which torch evaluates in its default float32: both factors are rounded to
    float32, the product is rounded to float32 (round to nearest even), and the
    ceiling is taken of that. Reproduced here with NumPy float32 scalars, whose
    multiply is IEEE round-to-nearest. (Example: c=50, budget=0.30 gives 16,
    where exact arithmetic gives 15.)
    """
    c32 = np.asarray(per_row).astype(np.float32)
    prod = c32 * np.float32(budget)
    assert prod.dtype == np.float32
    return np.ceil(prod).astype(np.int64)


def _as_tiles(x, nq, nk):
    if x is None:
        return None
    x = np.asarray(x)
    if x.ndim == 2:
        x = x[None, None]
    assert x.shape[-2:] == (nq, nk), (x.shape, nq, nk)
    return x.astype(bool)


def selection_plan(spec: SparseSpec, nq: int, nk: int, pins=None, drops=None):
    """selector.py, ``selection_plan``.

    must = diagonal | pins; forbidden = drops; candidates = ~must & ~forbidden;
    per_row = number of candidates; keep_per_row = ceil(per_row * budget)
    (float32, see ``budget_count``); covers_everything = every row may keep
    all its candidates. Shapes broadcast to (B or 1, H or 1, NQ, NK); the
    per-row counts have a trailing axis of length 1.
    """
    must = diagonal_blocks(nq, nk, spec.block_q, spec.block_kv)[None, None]
    p = _as_tiles(pins, nq, nk)
    d = _as_tiles(drops, nq, nk)
    if p is not None:
        must = must | p
    forbidden = d if d is not None else np.zeros_like(must)
    candidates = ~must & ~forbidden
    per_row = candidates.sum(axis=-1, keepdims=True).astype(np.int64)
    keep_per_row = budget_count(per_row, spec.budget)
    covers_everything = bool(np.all(keep_per_row >= per_row))
    return must, forbidden, candidates, keep_per_row, covers_everything


def select_blocks(q, k, spec: SparseSpec, pins=None, drops=None, return_scores=False):
    """selector.py, ``select_blocks``.

    Returns the int8 keep tensor (B, Hs, NQ, NK), or None when the plan covers
    every candidate and ``force`` is off (the caller then attends densely and
    drops are not applied). Otherwise: non-candidates score -inf; each row is
    ordered by score descending with ties in ascending kv index (a stable
    descending sort); a candidate is kept when its rank is below the row's
    budget count; must tiles are added and forbidden tiles removed last.
    With ``return_scores`` the float64 scores and the plan come back as well.
    The pooling step is ``pool_blocks``; the rest is ``select_pooled``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    return select_pooled(pool_blocks(q, spec.block_q), pool_blocks(k, spec.block_kv), spec, pins, drops,
                         return_scores)


def select_pooled(pq, pk, spec: SparseSpec, pins=None, drops=None, return_scores=False):
    """``select_blocks`` from the pooled tensors on: pq (B, Hq, NQ, D) and pk
    (B, Hkv, NK, D) as ``pool_blocks`` gives them. The head handling of
    ``score_blocks`` (``head_map``), the unscaled scores, the plan and the
    ranking, with the same results and return values as ``select_blocks``."""
    pq = np.asarray(pq, dtype=np.float64)
    pk = np.asarray(pk, dtype=np.float64)
    nq, nk = pq.shape[-2], pk.shape[-2]
    must, forbidden, cand, kpr, covers = selection_plan(spec, nq, nk, pins, drops)
    if covers and not spec.force:
        return (None, None, None) if return_scores else None
    hq, hk = head_map(pq, pk, spec.head_shared)
    scores = np.matmul(hq, np.swapaxes(hk, -1, -2))
    shape = scores.shape
    cand_b = np.broadcast_to(cand, shape)
    masked = np.where(cand_b, scores, -np.inf)
    # stable sort of the negated scores = descending, ties to the lower index
    order = np.argsort(-masked, axis=-1, kind="stable")
    rank = np.empty_like(order)
    np.put_along_axis(rank, order, np.broadcast_to(np.arange(nk), shape), axis=-1)
    keep = np.broadcast_to(must, shape) | ((rank < np.broadcast_to(kpr, shape[:-1] + (1,))) & cand_b)
    keep = keep & ~np.broadcast_to(forbidden, shape)
    keep = keep.astype(np.int8)
    if return_scores:
        plan = dict(must=must, forbidden=forbidden, candidates=cand,
                    keep_per_row=kpr, covers_everything=covers)
        return keep, scores, plan
    return keep


def boundary_scores(scores_row: np.ndarray, cand_row: np.ndarray, k: int):
    """The k-th and (k+1)-th highest candidate scores of one row, in the
    select order (score descending, kv index ascending), or None where the
    row has no such boundary (k == 0 or k == number of candidates).
    Used by the keep parity rule, which tolerates differences only between
    near-tied boundary scores."""
    c = int(cand_row.sum())
    if k <= 0 or k >= c:
        return None
    s = np.sort(scores_row[cand_row.astype(bool)])[::-1]
    return float(s[k - 1]), float(s[k])


def keep_to_lists(keep: np.ndarray):
    """Compacted kept-tile lists of a keep tensor: per row the count and the
    kept kv tile indices in ascending order (the column-index form a
    block-sparse attention reads in its inner loop, as in flex-attention's
    block mask discussed in attention-gym issue #56). Returns
    (count (..., NQ) int32, index (..., NQ, NK) int32 padded with -1)."""
    keep = np.asarray(keep).astype(bool)
    count = keep.sum(axis=-1).astype(np.int32)
    index = np.full(keep.shape, -1, dtype=np.int32)
    it = np.ndindex(*keep.shape[:-1])
    for pos in it:
        js = np.nonzero(keep[pos])[0]
        index[pos][: len(js)] = js
    return count, index


def radial_blocks(seq_q: int, seq_kv: int, density: float, spec: SparseSpec, return_width: bool = False):
    """selector.py, ``radial_blocks``: a static band around the diagonal.

    Tile centres are ((i+0.5)*bq, (j+0.5)*bkv); the band keeps tiles whose
    centre distance is at most w, with w found by 40 bisection steps on
    [0, max(seq_q, seq_kv)] so that the kept fraction reaches ``density``
    (the fraction is evaluated in float32, as the page does). Returns int8
    (1, 1, NQ, NK), and with ``return_width`` also w (the bisection's upper
    end)."""
    nq, nk = block_count(seq_q, spec.block_q), block_count(seq_kv, spec.block_kv)
    qc = (np.arange(nq, dtype=np.float64)[:, None] + 0.5) * spec.block_q
    kc = (np.arange(nk, dtype=np.float64)[None, :] + 0.5) * spec.block_kv
    dist = np.abs(qc - kc)
    low, high = 0.0, float(max(seq_q, seq_kv))
    for _ in range(40):
        mid = (low + high) / 2
        frac = float(np.mean((dist <= mid).astype(np.float32), dtype=np.float32))
        if frac < density:
            low = mid
        else:
            high = mid
    keep = (dist <= high).astype(np.int8)[None, None]
    return (keep, high) if return_width else keep


def schedule(steps: int, budget: float, bump: float = 0.0, bump_steps: int = 0):
    """selector.py, ``schedule``: per-step budgets. With a bump, the first and
    last min(bump_steps, ceil(steps/2)) steps use min(1, budget + bump); all
    others use ``budget``. At most two distinct values."""
    if bump <= 0 or bump_steps <= 0 or steps <= 0:
        return tuple([budget] * max(steps, 0))
    raised = min(1.0, budget + bump)
    edge = min(bump_steps, math.ceil(steps / 2))
    return tuple(raised if (i < edge or i >= steps - edge) else budget for i in range(steps))


def _f64(x):
    """float64 NumPy copy of an array slice (NumPy or torch, any float dtype)."""
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def select_rows(q, k, spec: SparseSpec, rows, pins=None, drops=None):
    """``select_blocks`` restricted to the listed keep rows, for inputs too
    large to score in full.

    ``rows`` are (b, h, i) indices into the (B, Hs, NQ, NK) keep. The plan
    (diagonal, pins, drops, per-row budget count and the dense short circuit)
    is the same as ``selection_plan``'s; for each row the pooled query vector
    and the pooled keys of its key head (or their means over heads when
    head_shared) are formed from the token slices it needs, then the row is
    ranked exactly as ``select_blocks`` ranks it. ``q`` and ``k`` may be
    NumPy or torch arrays of any float dtype. Returns None for the dense short
    circuit, else a dict mapping each row to (keep (NK,) int8, scores (NK,)
    float64, candidates (NK,) bool, k int).
    """
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    nq, nk = block_count(Sq, spec.block_q), block_count(Skv, spec.block_kv)
    must, forb, cand, kpr, covers = selection_plan(spec, nq, nk, pins, drops)
    if covers and not spec.force:
        return None
    g = Hq // Hkv
    pk_cache = {}

    def pooled_k(b, hk):
        key = (b, hk)
        if key not in pk_cache:
            if spec.head_shared:
                pk_cache[key] = np.mean([pool_blocks(_f64(k[b, hh]), spec.block_kv) for hh in range(Hkv)], axis=0)
            else:
                pk_cache[key] = pool_blocks(_f64(k[b, hk]), spec.block_kv)
        return pk_cache[key]

    def pooled_q(b, h, i):
        lo, hi = i * spec.block_q, min((i + 1) * spec.block_q, Sq)
        if spec.head_shared:
            return np.mean([_f64(q[b, hh, lo:hi]).sum(axis=0) / float(hi - lo) for hh in range(Hq)], axis=0)
        return _f64(q[b, h, lo:hi]).sum(axis=0) / float(hi - lo)

    def at(a, b, h, i):
        return a[0 if a.shape[0] == 1 else b, 0 if a.shape[1] == 1 else h, i]

    out = {}
    for (b, h, i) in rows:
        hk = 0 if spec.head_shared else h // g
        s = pooled_k(b, hk) @ pooled_q(b, h, i)
        c = at(cand, b, h, i)
        kk = int(at(kpr, b, h, i)[0])
        masked = np.where(c, s, -np.inf)
        order = np.argsort(-masked, kind="stable")
        rank = np.empty(nk, dtype=np.int64)
        rank[order] = np.arange(nk)
        keep = (at(must, b, h, i) | ((rank < kk) & c)) & ~at(forb, b, h, i)
        out[(b, h, i)] = (keep.astype(np.int8), s, c.copy(), kk)
    return out
