"""Seeded synthetic workloads for fixed-budget block-sparse attention.

This module is shared by the CPU oracle, the GPU tests and the bench. It holds
shapes, the seeded value recipes and the caller-side pin/drop patterns only;
none of the selection or attention arithmetic lives here.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)`` in
float32 and then rounded to bfloat16, so both sides see identical bits.
"N(mu, sigma)" means mean mu and standard deviation sigma (``randn * sigma``).

The five named workloads follow the configurations the selector is exercised
on (fixed-budget block selection, ``SparseSpec`` defaults block_q=128,
block_kv=64 in automatic/modules/attention/sparse/selector.py). The ``*_small``
variants keep each workload's structure at sizes the float64 oracle finishes in
seconds, and the ``ragged_*`` variants add partial final tiles, which none of
the five named workloads has.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_inputs", "morton_decode",
           "tile_counts", "pins_drops"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    D: int
    budget: float
    block_q: int = 128
    block_kv: int = 64
    head_shared: bool = False
    force: bool = False
    # value recipe: "iid", "segment_mean", "centroids", "fourier2d"
    recipe: str = "iid"
    # caller-side tile patterns: "none" or "sinks2_blockcausal"
    pins_drops: str = "none"
    params: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def NQ(self) -> int:
        return (self.Sq + self.block_q - 1) // self.block_q

    @property
    def NK(self) -> int:
        return (self.Skv + self.block_kv - 1) // self.block_kv

    @property
    def Hs(self) -> int:
        return 1 if self.head_shared else self.Hq

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def tile_counts(wl: Workload) -> tuple[int, int]:
    return wl.NQ, wl.NK


_W = [
    # 1. Tiny: i.i.d. N(0,1), per-head scoring, force on.
    Workload("tiny", B=1, Hq=2, Hkv=2, Sq=1024, Skv=1024, D=64, budget=0.30,
             force=True),
    # 2. GQA: N(0,1) plus a per-(batch, 512-token segment) vector N(0, 0.5)
    #    added to both Q and K, shared by every head.
    Workload("gqa", B=2, Hq=16, Hkv=4, Sq=8192, Skv=8192, D=128, budget=0.30,
             recipe="segment_mean", params={"segment": 512, "sigma": 0.5}),
    # 3. Head-shared long: Q and K = centroid + N(0,1); 64 centroids N(0,1)
    #    shared by all heads, one centroid per (batch, 256-token run).
    Workload("head_shared", B=1, Hq=32, Hkv=8, Sq=32768, Skv=32768, D=128,
             budget=0.10, head_shared=True, recipe="centroids",
             params={"run": 256, "n_centroids": 64, "centroid_scale": 1.0}),
    # 4. Cross-length: sinks (kv tiles 0 and 1) pinned, block-causal drops.
    Workload("cross", B=4, Hq=8, Hkv=8, Sq=4096, Skv=16000, D=64, budget=0.25,
             pins_drops="sinks2_blockcausal"),
    # 5. Large 2D-local: 256x512 grid in Morton order, 16 random Fourier modes
    #    of grid position plus N(0, 0.3) noise for Q and K; V ~ N(0,1).
    Workload("large2d", B=1, Hq=64, Hkv=8, Sq=131072, Skv=131072, D=128,
             budget=0.05, recipe="fourier2d",
             params={"rows": 256, "cols": 512, "modes": 16, "fmax": 1.0 / 32,
                     "noise": 0.3}),
]

# Oracle-sized variants with the same structure (several tiles, GQA, pins,
# drops, head sharing), plus ragged tails the named workloads lack.
_W += [
    Workload("gqa_small", B=1, Hq=4, Hkv=2, Sq=2048, Skv=2048, D=128,
             budget=0.30, recipe="segment_mean",
             params={"segment": 512, "sigma": 0.5}),
    Workload("head_shared_small", B=1, Hq=4, Hkv=2, Sq=2048, Skv=2048, D=128,
             budget=0.10, head_shared=True, recipe="centroids",
             params={"run": 256, "n_centroids": 64, "centroid_scale": 1.0}),
    Workload("cross_small", B=2, Hq=2, Hkv=2, Sq=1024, Skv=4000, D=64,
             budget=0.25, pins_drops="sinks2_blockcausal"),
    Workload("large2d_small", B=1, Hq=4, Hkv=2, Sq=4096, Skv=4096, D=128,
             budget=0.05, recipe="fourier2d",
             params={"rows": 64, "cols": 64, "modes": 16, "fmax": 1.0 / 32,
                     "noise": 0.3}),
    # ragged: partial final q tile and partial final kv tile
    Workload("ragged", B=1, Hq=2, Hkv=1, Sq=1000, Skv=1990, D=128,
             budget=0.30),
    Workload("ragged_cross", B=1, Hq=2, Hkv=2, Sq=4000, Skv=15990, D=64,
             budget=0.25, pins_drops="sinks2_blockcausal"),
    # a single, partial query tile
    Workload("nq1", B=1, Hq=2, Hkv=2, Sq=100, Skv=700, D=64, budget=0.30,
             force=True),
    # budget 1.0 with force: every tile kept, i.e. dense attention
    Workload("dense_force", B=1, Hq=2, Hkv=2, Sq=512, Skv=768, D=64,
             budget=1.0, force=True),
    # long rows (a head's pooled keys above 64 KB, as in the Large-2D
    # workload): scores on the tensor cores; per-head, ragged with pins and
    # drops, and head-shared
    Workload("long_kv_small", B=1, Hq=4, Hkv=2, Sq=1024, Skv=16384, D=128,
             budget=0.20),
    Workload("long_kv_ragged", B=2, Hq=2, Hkv=1, Sq=1000, Skv=20000, D=64,
             budget=0.15, pins_drops="sinks2_blockcausal"),
    Workload("long_kv_hs", B=1, Hq=4, Hkv=2, Sq=512, Skv=16384, D=128,
             budget=0.10, head_shared=True),
    # rows of 2048 kv tiles, as in the Large-2D workload (the longest rows
    # the register top-k holds), at a size the oracle selects in full
    Workload("long_kv_2k", B=1, Hq=2, Hkv=1, Sq=1024, Skv=131072, D=64,
             budget=0.05),
    # rows past 2048 kv tiles (the scores chunked through shared memory):
    # 4096 per head, and 8192 (the longest selection row) head-shared with a
    # partial last kv tile
    # more fused-selection CTAs (B x Hq x NQ/8 = 1024) than fit on the device
    # at once: the keys are then pooled by their own kernel before the select
    Workload("gqa_wide", B=8, Hq=64, Hkv=8, Sq=2048, Skv=2048, D=128,
             budget=0.30, recipe="segment_mean", params={"segment": 512, "sigma": 0.5}),
    Workload("long_kv_4k", B=1, Hq=2, Hkv=1, Sq=512, Skv=262144, D=128,
             budget=0.05),
    Workload("long_kv_8k_hs", B=1, Hq=2, Hkv=2, Sq=384, Skv=524263, D=64,
             budget=0.02, head_shared=True),
    # one kv group of the Large 2D-local workload (8 query heads, 1/8 of its
    # work), for profiling captures that must stay small; per kv group the
    # kernels see the same shapes, statistics and schedule
    Workload("large2d_1kv", B=1, Hq=8, Hkv=1, Sq=131072, Skv=131072, D=128,
             budget=0.05, recipe="fourier2d",
             params={"rows": 256, "cols": 512, "modes": 16, "fmax": 1.0 / 32,
                     "noise": 0.3}),
]

WORKLOADS = {w.name: w for w in _W}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def morton_decode(codes: np.ndarray, rows: int, cols: int) -> tuple[np.ndarray, np.ndarray]:
    """Grid position (x, y) of each Morton (Z-order) code.

    Bits are interleaved x0 y0 x1 y1 ... from the least significant end; when
    the grid is wider than tall (cols = 2*rows) the top bit is the extra x bit.
    For a 256x512 grid: bit 2i is x_i and bit 2i+1 is y_i for i < 8, bit 16 is
    x_8. The map is a bijection onto [0, rows*cols).
    """
    codes = np.asarray(codes, dtype=np.int64)
    ybits = int(math.log2(rows))
    xbits = int(math.log2(cols))
    assert (1 << ybits) == rows and (1 << xbits) == cols and xbits >= ybits
    x = np.zeros_like(codes)
    y = np.zeros_like(codes)
    pos = 0
    for i in range(max(xbits, ybits)):
        if i < xbits:
            x |= ((codes >> pos) & 1) << i
            pos += 1
        if i < ybits:
            y |= ((codes >> pos) & 1) << i
            pos += 1
    return x, y


def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


def _iid(g, B, H, S, D):
    return torch.randn(B, H, S, D, generator=g, dtype=torch.float32)


def pins_drops(wl: Workload):
    """Caller tile patterns, broadcast shape (1, 1, NQ, NK), int8.

    sinks2_blockcausal: pins are kv tiles {0, 1}; a kv tile j is dropped when it
    starts strictly after the query tile's end position scaled to the kv
    length: 64*j*Sq > (i+1)*128*Skv, evaluated in exact integers.
    """
    if wl.pins_drops == "none":
        return None, None
    assert wl.pins_drops == "sinks2_blockcausal"
    NQ, NK = wl.NQ, wl.NK
    pins = np.zeros((1, 1, NQ, NK), dtype=np.int8)
    pins[..., :, : min(2, NK)] = 1
    i = np.arange(NQ, dtype=np.int64)[:, None]
    j = np.arange(NK, dtype=np.int64)[None, :]
    drops = (wl.block_kv * j * wl.Sq > (i + 1) * wl.block_q * wl.Skv)
    return pins, drops.astype(np.int8)[None, None]


def upstream_grad(wl: Workload, seed: int = 0) -> torch.Tensor:
    """Seeded upstream gradient dO (B, Hq, Sq, D) for the backward: N(0, 1)
    rounded to bf16 (CPU)."""
    g = torch.Generator().manual_seed(2000 + seed)
    return _bf16(_iid(g, wl.B, wl.Hq, wl.Sq, wl.D))


def key_mask(wl: Workload, kind: str, seed: int = 0, per_head: bool = True) -> np.ndarray:
    """Seeded key-token mask, bool (B, Hkv or 1, Skv), True = takes part.

    ``random50``: every token kept with probability 1/2, independently (the
    50% patch masking of MaskDiT that NATTEN issue #124 discusses).
    ``padding``: per batch (and head when ``per_head``) a valid prefix of a
    random length in [Skv/4, Skv], the rest masked (a padded canvas).
    ``head0_off``: as ``random50`` but kv head 0 of batch 0 masked entirely.
    ``prefix_off``: the first 3*64 + 17 tokens masked, the rest kept.
    """
    g = np.random.default_rng(1000 + seed)
    H = wl.Hkv if per_head else 1
    shape = (wl.B, H, wl.Skv)
    if kind in ("random50", "head0_off"):
        m = g.random(shape) < 0.5
        if kind == "head0_off":
            m[0, 0] = False
    elif kind == "padding":
        lens = g.integers(wl.Skv // 4, wl.Skv + 1, size=shape[:2])
        m = np.arange(wl.Skv)[None, None, :] < lens[..., None]
    elif kind == "prefix_off":
        m = np.ones(shape, dtype=bool)
        m[..., : min(wl.Skv, 3 * 64 + 17)] = False
    else:
        raise ValueError(kind)
    return m


def make_inputs(wl: Workload, seed: int = 0, heads=None):
    """Seeded synthetic inputs for ``wl``.

    Returns a dict with ``q`` (B,Hq,Sq,D), ``k`` and ``v`` (B,Hkv,Skv,D) as
    CPU bfloat16 tensors, and ``pins``/``drops`` as int8 numpy arrays of
    broadcast shape (1,1,NQ,NK) or None.
    """
    g = torch.Generator().manual_seed(seed)
    B, Hq, Hkv, Sq, Skv, D = wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Skv, wl.D
    p = wl.params
    if wl.recipe == "iid":
        q = _bf16(_iid(g, B, Hq, Sq, D))
        k = _bf16(_iid(g, B, Hkv, Skv, D))
        v = _bf16(_iid(g, B, Hkv, Skv, D))
    elif wl.recipe == "segment_mean":
        seg, sigma = p["segment"], p["sigma"]
        assert Sq == Skv
        nseg = (Sq + seg - 1) // seg
        q = _iid(g, B, Hq, Sq, D)
        k = _iid(g, B, Hkv, Skv, D)
        v = _bf16(_iid(g, B, Hkv, Skv, D))
        mean = torch.randn(B, nseg, D, generator=g) * sigma
        tok = mean.repeat_interleave(seg, dim=1)[:, :Sq]  # (B, S, D)
        q = _bf16(q + tok[:, None])
        k = _bf16(k + tok[:, None])
    elif wl.recipe == "centroids":
        run, nc, cs = p["run"], p["n_centroids"], p["centroid_scale"]
        assert Sq == Skv
        nrun = (Sq + run - 1) // run
        bank = torch.randn(nc, D, generator=g) * cs
        assign = torch.randint(0, nc, (B, nrun), generator=g)
        tok = bank[assign].repeat_interleave(run, dim=1)[:, :Sq]  # (B,S,D)
        q = _bf16(_iid(g, B, Hq, Sq, D) + tok[:, None])
        k = _bf16(_iid(g, B, Hkv, Skv, D) + tok[:, None])
        v = _bf16(_iid(g, B, Hkv, Skv, D))
    elif wl.recipe == "fourier2d":
        q, k, v = _fourier2d(wl, g)
    else:
        raise ValueError(wl.recipe)
    pins, drops = pins_drops(wl)
    return {"q": q, "k": k, "v": v, "pins": pins, "drops": drops}


def _fourier2d(wl: Workload, g: torch.Generator):
    """Q/K features: per kv head and channel, a sum of random 2D Fourier modes.

    F[h, t, d] = sum_m cos(2*pi*(u_m*x_t + v_m*y_t) + phi[h, d, m]) with
    (u_m, v_m) ~ U[-fmax, fmax]^2 shared by all heads and channels and
    phi ~ U[0, 2*pi); (x_t, y_t) is the grid cell of Morton code t. Query head
    h uses the field of kv head h // (Hq/Hkv), so queries and keys are locally
    correlated. Q and K each add independent N(0, noise) noise; V ~ N(0,1).
    The sum is evaluated through cos(a+phi) = cos a cos phi - sin a sin phi.
    """
    p = wl.params
    B, Hq, Hkv, S, D = wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.D
    assert wl.Sq == wl.Skv == p["rows"] * p["cols"]
    M = p["modes"]
    fmax = p["fmax"]
    uv = (torch.rand(M, 2, generator=g, dtype=torch.float64) * 2 - 1) * fmax
    phi = torch.rand(B, Hkv, D, M, generator=g, dtype=torch.float64) * (2 * math.pi)
    x, y = morton_decode(np.arange(S), p["rows"], p["cols"])
    xt = torch.from_numpy(x).to(torch.float64)
    yt = torch.from_numpy(y).to(torch.float64)
    ang = 2 * math.pi * (xt[:, None] * uv[None, :, 0] + yt[:, None] * uv[None, :, 1])  # (S,M)
    ca, sa = torch.cos(ang), torch.sin(ang)
    grp = Hq // Hkv
    q = torch.empty(B, Hq, S, D, dtype=torch.bfloat16)
    k = torch.empty(B, Hkv, S, D, dtype=torch.bfloat16)
    fields = torch.empty(B, Hkv, S, D, dtype=torch.float32)
    for b in range(B):
        for h in range(Hkv):
            f = ca @ torch.cos(phi[b, h]).T - sa @ torch.sin(phi[b, h]).T  # (S, D)
            fields[b, h] = f.to(torch.float32)
    noise = p["noise"]
    for b in range(B):
        for h in range(Hkv):
            k[b, h] = _bf16(fields[b, h] + torch.randn(S, D, generator=g) * noise)
    for b in range(B):
        for h in range(Hq):
            q[b, h] = _bf16(fields[b, h // grp] + torch.randn(S, D, generator=g) * noise)
    v = _bf16(_iid(g, B, Hkv, S, D))
    return q, k, v
