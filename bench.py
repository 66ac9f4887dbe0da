#!/usr/bin/env python
"""Benchmark of the fixed-budget block-sparse attention path on B200.

One step = one pass of the whole path over one batch of synthetic input,
through the library's C ABI (nsa_forward): pool q and k, score + plan +
top-k keep (selector.py's select_blocks), attention over the kept tiles.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload large2d]
    python bench.py --impl reference ...      # the CPU oracle, timed alone

The headline workload is the largest one-GPU configuration, Large 2D-local
(B=1, Hq=64, Hkv=8, S=131072, D=128, budget 0.05). Its line carries:
- value: kept-tile attention TFLOP/s over the whole step (4*block_q*
  block_kv*D FLOPs per kept tile per query head), steps timed with CUDA
  events around each step, the L2 flushed before every step;
- attn / selection: the attention kernel's TFLOP/s and the selection's GB/s
  (q + k read, keep written, pin/drop masks read, timed as one span from
  before pooling to after selection so its kernels overlap as in a step),
  each also as a fraction of the measured peaks; roofline: the attention
  kernel against the bf16 tensor peak: the sustained one (a GEMM held under
  the power cap) when the power cap was active during the timed steps, else
  the burst one, with the fraction of the burst peak always beside it;
- e2e: the same metric through nsa_forward from pinned host buffers, every
  step copying q, k, v in and O, LSE out (copy-in, compute and copy-out on
  three streams over two device buffer sets; the single-stream figure is
  reported beside it);
- radial_control, key_mask, backward: the band control, the key-token mask
  and the backward over the same kept tiles;
- cpu_baseline: the CPU oracle on a bounded sample of the same workload, its
  time extrapolated to the whole step;
- configs: the same attention and selection figures (and the oracle's) for
  all five workloads: Tiny, GQA, Head-shared, Cross and Large 2D.

The L2 (126 MB) is flushed before every timed step by writing a 256 MiB
buffer and then reading another 256 MiB buffer, so that the flush's dirty
lines are written back before the step starts. Multi-GPU runs (torchrun) are
weak scaling: every rank processes its own independent batch (seed = rank);
there is no collective on the data path.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "block-sparse attn TFLOP/s (kept tiles) + selection GB/s; % of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
CONFIG_ORDER = ("tiny", "gqa", "head_shared", "cross", "large2d")


# ----------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tile_flops(wl) -> float:
    """4 * block_q * block_kv * D: the attention FLOPs of one kept tile for
    one query head."""
    return 4.0 * wl.block_q * wl.block_kv * wl.D


def kept_tile_flops(keep: torch.Tensor, wl) -> float:
    """4 * block_q * block_kv * D per kept tile per query head."""
    kept = float(keep.sum(dtype=torch.int64).item())
    heads_per_keep_row = wl.Hq if keep.shape[1] == 1 else 1
    return kept * heads_per_keep_row * tile_flops(wl)


def selection_bytes(wl, pins, drops) -> float:
    """Algorithmic bytes of pooling + selection: q and k read once (bf16),
    the int8 keep written, the pin/drop masks read."""
    b = wl.B * wl.Hq * wl.Sq * wl.D * 2 + wl.B * wl.Hkv * wl.Skv * wl.D * 2
    b += wl.B * wl.Hs * wl.NQ * wl.NK
    for m in (pins, drops):
        if m is not None:
            b += m.numel()
    return float(b)


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 100):
        self.index = index
        self.period = period_ms
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append({"sm": float(f[1]), "max": float(f[2]), "power": float(f[3]),
                             "hw_slowdown": f[5], "hw_thermal": f[6], "sw_thermal": f[7], "sw_power_cap": f[8]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw_slowdown", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power_cap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


def dist_setup(backend: str):
    """(rank, world, local_rank) from the torchrun environment; initialises
    the process group for world > 1 with a short timeout."""
    import datetime
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not torch.distributed.is_initialized():
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return rank, world, local


def barrier(world: int, device=None):
    if world > 1:
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank draws an independent batch of the same workload."""
    return rank


# ---------------------------------------------------------- oracle timing

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_units(wl):
    """The oracle's selection units: (batch, kv head) for per-head scoring
    (the query heads of one kv group are scored against its keys), one batch
    with all heads for head-shared scoring (the head means need every head)."""
    if wl.head_shared:
        return [(b, None) for b in range(wl.B)]
    return [(b, hk) for b in range(wl.B) for hk in range(wl.Hkv)]


def oracle_unit(wl, inp, unit, n_tiles, rng):
    """One unit of the oracle's path, timed in two parts: selection
    (select_blocks) over every query tile of the unit's heads, then attention
    (attention_tiles) for up to ``n_tiles`` seeded query tiles of those heads
    (every tile when the unit has no more). The bf16 -> float64 conversion of
    the inputs is not timed. Returns (selection s, attention s, attention
    FLOPs of the tiles done, tiles done, tiles in the unit)."""
    import oracle
    b, hk = unit
    g = wl.Hq // wl.Hkv
    spec = oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    if hk is None:
        qs, ks, vs = (inp[x][b:b + 1].double().numpy() for x in "qkv")
        heads = list(range(wl.Hq))
    else:
        qs = inp["q"][b:b + 1, hk * g:(hk + 1) * g].double().numpy()
        ks, vs = (inp[x][b:b + 1, hk:hk + 1].double().numpy() for x in "kv")
        heads = list(range(g))
    t0 = time.perf_counter()
    keep = oracle.select_blocks(qs, ks, spec, inp["pins"], inp["drops"])
    t_sel = time.perf_counter() - t0
    if keep is None:
        keep = np.ones((1, 1, wl.NQ, wl.NK), np.int8)
    all_tiles = [(0, h, i) for h in heads for i in range(wl.NQ)]
    if len(all_tiles) <= n_tiles:
        tiles = all_tiles
    else:
        tiles = [all_tiles[t] for t in sorted(rng.choice(len(all_tiles), n_tiles, replace=False))]
    t0 = time.perf_counter()
    oracle.attention_tiles(qs, ks, vs, keep, wl.block_q, wl.block_kv, wl.scale, tiles)
    t_attn = time.perf_counter() - t0
    kept = sum(int(keep[0, 0 if keep.shape[1] == 1 else h, i].sum()) for (_, h, i) in tiles)
    return t_sel, t_attn, kept * tile_flops(wl), len(tiles), len(all_tiles)


def plan_kept_flops(wl, pins, drops) -> float:
    """The step's kept-tile FLOPs from the oracle's plan alone: every keep
    row keeps |must minus forbidden| + ceil(c * budget) tiles (all NK on the
    dense short circuit), each worth 4*block_q*block_kv*D per query head."""
    import oracle
    spec = oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    must, forb, _, kpr, covers = oracle.selection_plan(spec, wl.NQ, wl.NK, pins, drops)
    if covers and not wl.force:
        kept = np.full((wl.B, wl.Hs, wl.NQ), wl.NK)
    else:
        kept = np.broadcast_to((must & ~forb).sum(-1) + kpr[..., 0], (wl.B, wl.Hs, wl.NQ))
    heads_per_keep_row = wl.Hq // wl.Hs
    return float(kept.sum()) * heads_per_keep_row * tile_flops(wl)


def time_oracle(wl, inp, budget_s: float, flops_full: float, sel_bytes: float, n_tiles: int = 32):
    """The oracle on seeded (batch, kv head) units of ``wl`` for about
    ``budget_s`` seconds (at least one unit), its time extrapolated to the
    whole workload: selection seconds per unit times the number of units, and
    attention seconds per kept-tile FLOP times the step's kept-tile FLOPs.
    Returns the cpu_baseline record in the metric's unit."""
    units = oracle_units(wl)
    rng = np.random.default_rng(0)
    order = rng.permutation(len(units))
    t_sel = t_attn = fl = 0.0
    done = tiles_done = tiles_all = 0
    start = time.perf_counter()
    for u in order:
        s, a, f, nt, na = oracle_unit(wl, inp, units[u], n_tiles, rng)
        t_sel += s
        t_attn += a
        fl += f
        done += 1
        tiles_done += nt
        tiles_all += na
        if time.perf_counter() - start >= budget_s:
            break
    sel_full = t_sel / done * len(units)
    attn_full = t_attn / fl * flops_full if fl > 0 else 0.0
    step_s = sel_full + attn_full
    full = done == len(units) and tiles_done == tiles_all
    sample = (f"{done} of {len(units)} selection units ({'batch' if wl.head_shared else '(batch, kv head)'}: "
              f"select_blocks over all query tiles of its heads) and attention over {tiles_done} of their "
              f"{tiles_all} query tiles, {t_sel + t_attn:.1f} s of oracle time"
              + ("" if full else "; selection extrapolated per unit, attention per kept-tile FLOP"))
    return {"value": flops_full / step_s / 1e12 if step_s > 0 else None, "unit": "TFLOP/s (kept tiles)",
            "cores": blas_threads(), "kind": "oracle", "sample": sample,
            "extrapolated": not full, "step_s": round(step_s, 3),
            "selection_gbs": round(sel_bytes / sel_full / 1e9, 4) if sel_full > 0 else None,
            "selection_s": round(sel_full, 3), "attn_s": round(attn_full, 3), "host_cpus": os.cpu_count()}


# ------------------------------------------------------------ our arm

class Flusher:
    """Evicts the L2 between timed steps: writes one 256 MiB buffer, then
    reads another, so that the written lines are back in HBM before the step."""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def _ev():
    return torch.cuda.Event(enable_timing=True)


def bench_workload(nsa, name, args, dev, rank, world, peaks, headline: bool):
    """Times ``name`` on this rank. Every rank takes the same collective steps.
    Returns a dict with the line's fields for the workload (``headline`` adds
    the clocks, the extras, the end-to-end run and the launch count)."""
    wl = workloads.get(name)
    inp = workloads.make_inputs(wl, seed=rank_seed(rank))
    q, k, v = (inp[x].to(dev) for x in "qkv")
    pins = None if inp["pins"] is None else torch.from_numpy(inp["pins"]).to(dev)
    drops = None if inp["drops"] is None else torch.from_numpy(inp["drops"]).to(dev)
    spec = nsa.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    ws = nsa.workspace(wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Skv, wl.D, spec, dev)
    out = torch.empty_like(q)
    lse = torch.empty(wl.B, wl.Hq, wl.Sq, dtype=torch.float32, device=dev)
    keep = torch.empty(wl.B, wl.Hs, wl.NQ, wl.NK, dtype=torch.int8, device=dev)
    cold_l2 = Flusher(dev)
    steps = args.steps if headline else max(3, min(args.steps, args.config_steps))
    n_split = min(steps, 100)

    def step(events=None):
        nsa.nsa_forward(q, k, v, spec, wl.scale, pins, drops, keep_out=keep, out=out, lse=lse, ws=ws,
                        events=events)

    for _ in range(args.warmup):
        cold_l2()
        step()
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    flops_step = kept_tile_flops(keep, wl)
    sel_bytes = selection_bytes(wl, pins, drops)

    # whole steps, timed with the outer events only (the kernels are chained
    # by programmatic dependent launch, which a middle event would serialise)
    ev = [[_ev(), None, None, _ev()] for _ in range(steps)]
    clocks = ClockSampler(dev.index if dev.index is not None else 0) if headline else None
    barrier(world, dev)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)  # first sample before the timed region
    n0 = nsa.nsa_kernel_launches()
    for s in range(steps):
        cold_l2()
        step(ev[s])
    launches = nsa.nsa_kernel_launches() - n0
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    barrier(world, dev)
    nsa.nsa_device_status()
    t_step = [e[0].elapsed_time(e[3]) for e in ev]

    # per-kernel split (a separate loop; its boundaries are serialised by the
    # events), then selection as one span (pool + select with no event
    # between them, so that they overlap as inside a step)
    ev_split = [[_ev() for _ in range(4)] for _ in range(n_split)]
    for e in ev_split:
        cold_l2()
        step(e)
    ev_sel = [[_ev(), None, _ev(), None] for _ in range(n_split)]
    for e in ev_sel:
        cold_l2()
        step(e)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    t_pool = statistics.mean(e[0].elapsed_time(e[1]) for e in ev_split)
    t_sel = statistics.mean(e[1].elapsed_time(e[2]) for e in ev_split)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev_split)
    sel_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in ev_sel)

    total_ms = max_over_ranks(sum(t_step), world, dev)
    ms_per_step = total_ms / steps
    flops_all = sum_over_ranks(flops_step, world, dev)
    value = flops_all / (ms_per_step * 1e-3) / 1e12
    peak_t = float(peaks["bf16_tflops"])
    peak_h = float(peaks["hbm_gbs"])
    attn_tflops = flops_step / (attn_ms * 1e-3) / 1e12
    sel_gbs = sel_bytes / (sel_ms * 1e-3) / 1e9
    density = float(keep.sum(dtype=torch.int64).item()) / keep.numel()
    res = {
        "wl": wl, "steps": steps, "ms_per_step": ms_per_step, "value": value, "flops_step": flops_step,
        "flops_all": flops_all, "sel_bytes": sel_bytes, "attn_tflops": attn_tflops, "attn_ms": attn_ms,
        "sel_ms": sel_ms, "sel_gbs": sel_gbs, "pool_ms": t_pool, "select_ms": t_sel, "clocks": clk,
        "launches": launches, "n_split": n_split,
    }
    res["summary"] = {
        "shape": f"B{wl.B} Hq{wl.Hq} Hkv{wl.Hkv} Sq{wl.Sq} Skv{wl.Skv} D{wl.D} budget {wl.budget}"
                 + (" head_shared" if wl.head_shared else "") + (" pins+drops" if pins is not None else ""),
        "value_tflops": round(value, 3), "ms_per_step": round(ms_per_step, 5), "steps": steps,
        "kept_density": round(density, 6), "kept_tile_gflop": round(flops_step / 1e9, 3),
        "attn_tflops": round(attn_tflops, 2), "attn_ms": round(attn_ms, 5),
        "attn_frac_bf16_peak": round(attn_tflops / peak_t, 4),
        "selection_gbs": round(sel_gbs, 1), "selection_ms": round(sel_ms, 5), "selection_bytes": sel_bytes,
        "selection_frac_hbm": round(sel_gbs / peak_h, 4),
        "kernels_per_step": launches / steps,
    }

    if headline:
        res.update(headline_extras(nsa, wl, inp, q, k, v, pins, drops, spec, keep, out, lse, ws, cold_l2,
                                   flops_step, flops_all, density, n_split, args, dev, world, peak_t))

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle(wl, inp, args.cpu_seconds, flops_step, sel_bytes)
        res["summary"]["cpu_baseline"] = cpu
    return res


def headline_extras(nsa, wl, inp, q, k, v, pins, drops, spec, keep, out, lse, ws, cold_l2, flops_step,
                    flops_all, density, n_split, args, dev, world, peak_t):
    """Radial band control, key-token mask, backward and end to end for the
    headline workload."""
    res = {}
    # radial band control (selector.py radial_blocks: a fixed band around the
    # diagonal, the baseline a score-based selection should improve on): a
    # band keeping the same fraction of tiles as this selection, built on the
    # device, and the same attention kernel timed over it (the call includes
    # its keep-to-list conversion)
    rkeep, _, _, rwidth = nsa.nsa_radial_blocks(wl.B, wl.Sq, wl.Skv, density, spec, device=dev)
    rflops = kept_tile_flops(rkeep, wl)
    r_ev = [(_ev(), _ev()) for _ in range(n_split)]
    for it in range(args.warmup + n_split):
        cold_l2()
        e = r_ev[it - args.warmup] if it >= args.warmup else None
        if e:
            e[0].record()
        nsa.nsa_block_sparse_attn_fwd(q, k, v, rkeep, wl.scale, wl.block_q, wl.block_kv, out=out, lse=lse, ws=ws)
        if e:
            e[1].record()
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    r_ms = statistics.mean(a.elapsed_time(b) for a, b in r_ev)
    res["radial_control"] = {
        "density_target": round(density, 6),
        "density": round(float(rkeep.sum(dtype=torch.int64).item()) / rkeep.numel(), 6),
        "half_width_tokens": float(rwidth.item()), "attn_ms": round(r_ms, 5),
        "attn_tflops": round(rflops / (r_ms * 1e-3) / 1e12, 2),
        "note": "attention over a radial band keeping the selection's tile fraction; "
                "the time includes the keep-to-list conversion"}
    del rkeep

    # token-level key mask inside the kept tiles (NATTEN issue #124's
    # qkv_mask, True takes part): the selection's keep with half of the key
    # tokens masked at random, timed beside the unmasked call on the same keep
    # (both calls include their keep-to-list conversion)
    kmask = torch.from_numpy(workloads.key_mask(wl, "random50").astype(np.int8)).to(dev)
    m_ev = [[_ev() for _ in range(4)] for _ in range(n_split)]
    for it in range(args.warmup + n_split):
        e = m_ev[it - args.warmup] if it >= args.warmup else None
        cold_l2()
        if e:
            e[0].record()
        nsa.nsa_block_sparse_attn_fwd_masked(q, k, v, keep, kmask, wl.scale, wl.block_q, wl.block_kv,
                                             out=out, lse=lse, ws=ws)
        if e:
            e[1].record()
        cold_l2()
        if e:
            e[2].record()
        nsa.nsa_block_sparse_attn_fwd(q, k, v, keep, wl.scale, wl.block_q, wl.block_kv, out=out, lse=lse, ws=ws)
        if e:
            e[3].record()
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    km_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in m_ev)
    ku_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in m_ev)
    res["key_mask"] = {
        "kind": "random50", "kept_key_fraction": round(float(kmask.float().mean().item()), 4),
        "attn_ms": round(km_ms, 5), "unmasked_attn_ms": round(ku_ms, 5),
        "attn_tflops": round(flops_step / (km_ms * 1e-3) / 1e12, 2),
        "note": "FLOP/s counts the kept tiles' full tensor work (masking removes none of it); "
                "both times include the keep-to-list conversion"}
    del kmask

    # backward over the same kept tiles (dQ, dK, dV) for a seeded upstream
    # gradient, from this step's forward output and LSE
    nsa.nsa_forward(q, k, v, spec, wl.scale, pins, drops, keep_out=keep, out=out, lse=lse, ws=ws)
    dout = workloads.upstream_grad(wl).to(dev)
    bws = nsa.bwd_workspace(wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Skv, wl.D, wl.Hs, dev)
    gq, gk_, gv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    b_ev = [(_ev(), _ev()) for _ in range(n_split)]
    for it in range(args.warmup + n_split):
        cold_l2()
        e = b_ev[it - args.warmup] if it >= args.warmup else None
        if e:
            e[0].record()
        nsa.nsa_block_sparse_attn_bwd(q, k, v, out, lse, dout, keep, wl.scale, wl.block_q, wl.block_kv,
                                      dq=gq, dk=gk_, dv=gv, ws=bws)
        if e:
            e[1].record()
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    bwd_ms = statistics.mean(a.elapsed_time(b) for a, b in b_ev)
    bwd_flops = 2.5 * flops_step
    res["backward"] = {
        "ms": round(bwd_ms, 5), "tflops": round(bwd_flops / (bwd_ms * 1e-3) / 1e12, 2),
        "frac_of_bf16_peak": round(bwd_flops / (bwd_ms * 1e-3) / 1e12 / peak_t, 4),
        "note": "five products per kept tile and query head (S, dP, dV, dK, dQ), 2.5x the forward's "
                "count; the dQ kernel's recomputed S and dP are not counted; the time includes "
                "<dO, O>, both list conversions, the dK/dV kernel and the dQ kernel"}
    del dout, bws, gq, gk_, gv

    # end to end through the public API with host buffers: every step copies
    # its q, k, v in from pinned host memory and its output and LSE back.
    # First one stream, each step's copies and kernels in sequence; then the
    # way a serving loop runs it: copy-in, compute and copy-out on three
    # streams with two device buffer sets, so that step s+1's inputs and step
    # s-1's outputs cross PCIe while step s computes (the reported value).
    e2e_steps = max(3, args.e2e_steps)
    hq, hk_, hv = (t.pin_memory() for t in (inp["q"], inp["k"], inp["v"]))
    ho = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    hl = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
    e0, e1 = _ev(), _ev()
    ec = [_ev() for _ in range(4)]  # around the copies of the first timed step
    for it in range(1 + e2e_steps):
        if it == 1:
            barrier(world, dev)
            torch.cuda.synchronize()
            e0.record()
        if it == 1:
            ec[0].record()
        q.copy_(hq, non_blocking=True)
        k.copy_(hk_, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        if it == 1:
            ec[1].record()
        nsa.nsa_forward(q, k, v, spec, wl.scale, pins, drops, keep_out=keep, out=out, lse=lse, ws=ws)
        if it == 1:
            ec[2].record()
        ho[0].copy_(out, non_blocking=True)
        hl[0].copy_(lse, non_blocking=True)
        if it == 1:
            ec[3].record()
    e1.record()
    torch.cuda.synchronize()
    barrier(world, dev)
    serial_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    ref_o = ho[0].clone()

    bq_, bk_, bv_ = [q, torch.empty_like(q)], [k, torch.empty_like(k)], [v, torch.empty_like(v)]
    bo_, bl_ = [out, torch.empty_like(out)], [lse, torch.empty_like(lse)]
    s_in, s_c, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n_pipe = 2 + e2e_steps  # two untimed steps fill the pipeline
    ev_in = [torch.cuda.Event() for _ in range(n_pipe)]
    ev_c = [torch.cuda.Event() for _ in range(n_pipe)]
    ev_out = [torch.cuda.Event() for _ in range(n_pipe)]
    p0, p1 = _ev(), _ev()
    barrier(world, dev)
    torch.cuda.synchronize()
    for s_ in range(n_pipe):
        bf = s_ % 2
        if s_ == 2:
            # the timed steps' copies and kernels all follow this point: s_in
            # waits for steps 0 and 1 to finish before it records it
            s_in.wait_event(ev_out[1])
            p0.record(s_in)
        with torch.cuda.stream(s_in):
            if s_ >= 2:
                s_in.wait_event(ev_c[s_ - 2])  # step s-2 no longer reads this set
            bq_[bf].copy_(hq, non_blocking=True)
            bk_[bf].copy_(hk_, non_blocking=True)
            bv_[bf].copy_(hv, non_blocking=True)
            ev_in[s_].record(s_in)
        with torch.cuda.stream(s_c):
            s_c.wait_event(ev_in[s_])
            if s_ >= 2:
                s_c.wait_event(ev_out[s_ - 2])  # step s-2's output has left this set
            nsa.nsa_forward(bq_[bf], bk_[bf], bv_[bf], spec, wl.scale, pins, drops, keep_out=keep, out=bo_[bf],
                            lse=bl_[bf], ws=ws)
            ev_c[s_].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[s_])
            ho[bf].copy_(bo_[bf], non_blocking=True)
            hl[bf].copy_(bl_[bf], non_blocking=True)
            ev_out[s_].record(s_out)
    p1.record(s_out)
    torch.cuda.synchronize()
    barrier(world, dev)
    nsa.nsa_device_status()
    # the last step's output must equal the single-stream result; if it did
    # not, the single-stream figure is the one reported
    pipe_ok = torch.equal(ho[(n_pipe - 1) % 2], ref_o)
    if not pipe_ok:
        print("bench: pipelined end-to-end output differs; reporting the single-stream figure", file=sys.stderr)
    pipe_ms = max_over_ranks(p0.elapsed_time(p1), world, dev) / e2e_steps  # every rank takes this collective
    e2e_ms = pipe_ms if pipe_ok else serial_ms
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = ho[0].numel() * ho[0].element_size() + hl[0].numel() * hl[0].element_size()
    # the link's own rates, from the copies of one serial step (each alone on
    # the link): with copy-in and copy-out overlapped, a step cannot take
    # less than the longer of the two
    h2d_gbs = h2d / (ec[0].elapsed_time(ec[1]) * 1e-3) / 1e9
    d2h_gbs = d2h / (ec[2].elapsed_time(ec[3]) * 1e-3) / 1e9
    link_ms = max(h2d / h2d_gbs, d2h / d2h_gbs) / 1e6
    res["e2e"] = {
        "value": round(flops_all / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
        "schedule": ("copy-in, compute and copy-out on three streams, two device buffer sets" if pipe_ok
                     else "single stream"),
        "single_stream_ms_per_step": round(serial_ms, 4),
        "single_stream_value": round(flops_all / (serial_ms * 1e-3) / 1e12, 3),
        "link": {"h2d_gbs": round(h2d_gbs, 2), "d2h_gbs": round(d2h_gbs, 2), "bound_ms_per_step": round(link_ms, 3),
                 "frac": round(link_ms / e2e_ms, 4),
                 "note": "measured on this step's own copies, each direction alone; the bound is the longer "
                         "direction's time, the pipelined step's floor when the two directions overlap"}}
    return res


def load_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, if it was
    taken on the current attention source (else null)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "top_kv_tile_b200", "csrc", "attn_fwd.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    e = d.get(workload)
    if not e or e.get("attn_fwd_sha") != h:
        return None
    return e.get("dram_bytes_per_launch")


def run_ours(args):
    rank, world, local = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import top_kv_tile_b200 as nsa

    peaks, peak_src = load_peaks()
    peak_t = float(peaks["bf16_tflops"])
    head = bench_workload(nsa, args.workload, args, dev, rank, world, peaks, headline=True)
    configs = {}
    if not args.no_configs:
        for name in CONFIG_ORDER:
            if name == args.workload:
                configs[name] = head["summary"]
                continue
            torch.cuda.empty_cache()
            configs[name] = bench_workload(nsa, name, args, dev, rank, world, peaks, headline=False)["summary"]

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    wl = head["wl"]
    cpu = head["summary"].get("cpu_baseline")
    # the tensor peak paired with how the kernel ran: the sustained figure
    # (a GEMM held for seconds under the 1 kW power cap) when the power cap
    # was active during the timed steps, else the burst figure; the fraction
    # of the burst peak is kept beside it either way
    clk = head["clocks"] or {}
    capped = "sw_power_cap" in (clk.get("reasons") or [])
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak_t))
    roof_peak = peak_sus if capped else peak_t
    roofline = {
        "kernel": "attn_fwd_kernel", "bound": "tensor", "achieved": round(head["attn_tflops"], 2),
        "peak": roof_peak, "unit": "TFLOP/s", "frac": round(head["attn_tflops"] / roof_peak, 4),
        "peak_source": (f"{peak_src} bf16_tflops_sustained (sw_power_cap active during the timed steps)" if capped
                        else f"{peak_src} bf16_tflops (burst)"),
        "frac_of_burst": round(head["attn_tflops"] / peak_t, 4), "burst_peak": peak_t,
        "traffic": load_traffic(wl.name)}
    line = {
        "metric": METRIC,
        "value": round(head["value"], 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(head["ms_per_step"], 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "Sq": wl.Sq, "Skv": wl.Skv,
                   "D": wl.D, "block_q": wl.block_q, "block_kv": wl.block_kv, "budget": wl.budget,
                   "head_shared": wl.head_shared, "kept_tile_gflop_per_rank_step": round(head["flops_step"] / 1e9, 3),
                   "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)",
                   "parallelism": f"dp{world} (independent batches)"},
        "attn": {"tflops": round(head["attn_tflops"], 2), "ms": round(head["attn_ms"], 5),
                 "launches_timed": head["n_split"], "frac_bf16_peak": round(head["attn_tflops"] / peak_t, 4)},
        "selection": {"gbs": round(head["sel_gbs"], 1), "ms": round(head["sel_ms"], 5), "bytes": head["sel_bytes"],
                      "frac_hbm": round(head["sel_gbs"] / float(peaks["hbm_gbs"]), 4),
                      "pool_ms": round(head["pool_ms"], 5), "select_ms": round(head["select_ms"], 5)},
        "roofline": roofline,
        "e2e": head["e2e"],
        "radial_control": head["radial_control"],
        "key_mask": head["key_mask"],
        "backward": head["backward"],
        "cpu_baseline": cpu,
        "gpu_launches": head["launches"],
        "clocks": head["clocks"],
        "configs": configs,
        "peaks": {"hbm_gbs": float(peaks["hbm_gbs"]), "bf16_tflops": peak_t, "bf16_tflops_sustained": peak_sus,
                  "source": peak_src},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ reference arm

def run_reference(args):
    """The CPU oracle as the reference implementation, timed on the host's
    cores on the same workload: each step is one seeded selection unit
    ((batch, kv head), or a batch for head-shared scoring) plus attention
    over a few of its query tiles, and its time is extrapolated to the whole
    workload (selection per unit, attention per kept-tile FLOP). Under
    torchrun only rank 0 works; the others exit at once."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl = workloads.get(args.workload)
    inp = workloads.make_inputs(wl)
    units = oracle_units(wl)
    rng = np.random.default_rng(0)
    flops_full = plan_kept_flops(wl, inp["pins"], inp["drops"])
    n_tiles = 2
    for s in range(args.warmup):
        oracle_unit(wl, inp, units[s % len(units)], n_tiles, rng)
    step_s = []
    for s in range(args.steps):
        t_sel, t_attn, fl, _, _ = oracle_unit(wl, inp, units[s % len(units)], n_tiles, rng)
        step_s.append(t_sel * len(units) + (t_attn / fl * flops_full if fl > 0 else 0.0))
    ms = 1e3 * statistics.mean(step_s)
    value = flops_full / (ms * 1e-3) / 1e12
    sample = (f"per step: select_blocks for one {'batch' if wl.head_shared else '(batch, kv head)'} unit over all "
              f"query tiles + attention for {n_tiles} of its query tiles, cycling over the {len(units)} units; "
              f"the step time is extrapolated to the whole workload (selection per unit, attention per "
              f"kept-tile FLOP)")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "Sq": wl.Sq, "Skv": wl.Skv,
                   "D": wl.D, "block_q": wl.block_q, "block_kv": wl.block_kv, "budget": wl.budget,
                   "head_shared": wl.head_shared},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s (kept tiles)", "kind": "oracle",
                         "cores": blas_threads(), "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large2d", choices=sorted(workloads.WORKLOADS),
                    help="the headline workload (default: Large 2D-local, the largest one-GPU configuration)")
    ap.add_argument("--config-steps", type=int, default=20,
                    help="timed steps for each workload of the configs block (at most --steps)")
    ap.add_argument("--e2e-steps", type=int, default=40,
                    help="timed end-to-end steps (a separate measurement from the --steps kernel timing)")
    ap.add_argument("--cpu-seconds", type=float, default=6.0,
                    help="oracle seconds per workload for the CPU baseline (at least one unit)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="time the headline workload only")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        if world == 1:
            ap.error(f"--gpus {args.gpus} needs torchrun with {args.gpus} processes")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
