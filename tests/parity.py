"""Comparison rules between the CUDA path and the CPU oracle.

Keep flags: bit-exact per row, except in rows whose k-th and (k+1)-th oracle
candidate scores differ by less than 1e-5 relative (|s_k - s_k+1| <
1e-5 * max(|s_k|, |s_k+1|)). In such a row the two keeps may differ only on
tiles whose oracle score lies within that tolerance of s_k; the kept counts
must agree and every must-and-not-forbidden tile must be present.

Attention (computed from the same keep): bf16 output max-abs 2e-2, float32
LSE max-abs 1e-4.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle

TIE_RTOL = 1e-5
OUT_ATOL = 2e-2
LSE_ATOL = 1e-4


def _near(a, b):
    return abs(a - b) < TIE_RTOL * max(abs(a), abs(b))


def check_keep_row(pos, g, o, s, cand, k, must_not_forbidden):
    """One keep row: returns "exact" or "tie"; raises AssertionError on a
    violation of the rule in the module docstring."""
    g = np.asarray(g).astype(np.int8)
    o = np.asarray(o).astype(np.int8)
    if np.array_equal(g, o):
        return "exact"
    bd = oracle.boundary_scores(s, cand, k)
    assert bd is not None and _near(*bd), (
        f"keep row {pos} differs and its boundary scores {bd} are not a near tie")
    sk = bd[0]
    for j in np.nonzero(g != o)[0]:
        assert cand[j] and _near(float(s[j]), sk), (
            f"row {pos}: tile {j} (score {s[j]}) differs but is not tied with s_k={sk}")
    assert g.sum() == o.sum(), f"row {pos}: kept counts differ ({g.sum()} vs {o.sum()})"
    assert np.all(g[must_not_forbidden] == 1), f"row {pos}: a must tile is missing"
    return "tie"


def check_keep_rows(gpu_keep, ora_keep, scores, plan, rows=None):
    """Compare keep rows. ``rows``: iterable of (b, h, i) index tuples into
    the (B, Hs, NQ, NK) tensors (all rows when None). Returns a dict with the
    number of rows checked, exact rows and tie-tolerated rows; raises
    AssertionError on any violation."""
    gpu_keep = np.asarray(gpu_keep).astype(np.int8)
    ora_keep = np.asarray(ora_keep).astype(np.int8)
    shape = ora_keep.shape
    must = np.broadcast_to(plan["must"], shape)
    forb = np.broadcast_to(plan["forbidden"], shape)
    cand = np.broadcast_to(plan["candidates"], shape)
    kpr = np.broadcast_to(plan["keep_per_row"], shape[:-1] + (1,))
    if rows is None:
        rows = list(np.ndindex(*shape[:-1]))
    stats = {"rows": 0, "exact": 0, "tie_tolerated": 0}
    for pos in rows:
        stats["rows"] += 1
        r = check_keep_row(pos, gpu_keep[pos], ora_keep[pos], scores[pos], cand[pos], int(kpr[pos][0]),
                           must[pos] & ~forb[pos])
        stats["exact" if r == "exact" else "tie_tolerated"] += 1
    return stats


def check_lists(keep, count, index):
    """The compacted lists are the ascending kept indices of each keep row."""
    keep = np.asarray(keep).astype(bool)
    count = np.asarray(count)
    index = np.asarray(index).astype(np.int64) & 0xFFFF
    for pos in np.ndindex(*keep.shape[:-1]):
        js = np.nonzero(keep[pos])[0]
        assert count[pos] == len(js), (pos, count[pos], len(js))
        assert np.array_equal(index[pos][: len(js)], js), pos


def check_attention(out, lse, ref_o, ref_lse, out_atol=OUT_ATOL, lse_atol=LSE_ATOL):
    out = np.asarray(out, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin), "LSE finiteness differs (empty rows)"
    assert np.all(np.isneginf(lse[~fin])), "empty rows must have LSE = -inf"
    eo = float(np.max(np.abs(out - ref_o))) if out.size else 0.0
    el = float(np.max(np.abs(lse[fin] - ref_lse[fin]))) if fin.any() else 0.0
    assert eo <= out_atol, f"out max-abs error {eo} > {out_atol}"
    assert el <= lse_atol, f"LSE max-abs error {el} > {lse_atol}"
    return {"out_maxabs": eo, "lse_maxabs": el}


# Gradients from the backward: bf16 outputs of sums of bf16-rounded P and dS
# products accumulated in f32. Each product carries a relative rounding of
# 2^-9 (P or dS to bf16) and each output one more (its own rounding to
# bf16), so the relative Frobenius error of a gradient sits near 2^-9 and the
# error of its worst element near 2^-8 of the largest entry. The bounds are
# twice those figures; the largest errors measured over every case of
# tests/test_backward.py (the full-size GQA sample included) are 3.1e-3
# (Frobenius, dQ) and 5.0e-3 (max, dQ).
GRAD_REL_FRO = 2.0 * 2.0 ** -9
GRAD_REL_MAX = 2.0 * 2.0 ** -8


def check_grad(g, ref, name="grad", rel_fro=GRAD_REL_FRO, rel_max=GRAD_REL_MAX):
    g = np.asarray(g, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(g - ref))) if ref.size else 0.0
    nref = float(np.linalg.norm(ref))
    fro = float(np.linalg.norm(g - ref)) / nref if nref > 0 else float(np.linalg.norm(g))
    report = os.environ.get("NSA_GRAD_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"name": name, "rel_max": err / scale if scale > 0 else 0.0, "rel_fro": fro,
                                "test": os.environ.get("PYTEST_CURRENT_TEST", "")}) + "\n")
    assert err <= rel_max * scale + 1e-6, f"{name}: max-abs error {err} > {rel_max} x {scale}"
    assert fro <= rel_fro or nref == 0 and fro <= 1e-6, f"{name}: relative Frobenius error {fro} > {rel_fro}"
    return {"maxabs": err, "scale": scale, "rel_fro": fro}
