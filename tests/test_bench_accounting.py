"""The bench's accounting on the host: the algorithmic bytes of the selection,
the kept-tile FLOP count and the number of library kernels per step, against
counts worked out by hand from the workload shapes (no GPU needed)."""
import torch

import bench
import workloads


def test_selection_bytes_gqa_by_hand():
    # q: 2*16*8192*128 bf16 = 67,108,864 B; k: 2*4*8192*128 bf16 = 16,777,216 B;
    # keep: 2*16*64*128 int8 = 262,144 B
    wl = workloads.get("gqa")
    assert bench.selection_bytes(wl, None, None) == 67_108_864 + 16_777_216 + 262_144


def test_selection_bytes_counts_pin_and_drop_masks():
    wl = workloads.get("tiny")
    base = bench.selection_bytes(wl, None, None)
    pins = torch.zeros(1, 1, wl.NQ, wl.NK, dtype=torch.int8)
    drops = torch.zeros(1, 1, wl.NQ, wl.NK, dtype=torch.int8)
    assert bench.selection_bytes(wl, pins, drops) == base + 2 * wl.NQ * wl.NK


def test_kept_tile_flops_per_query_head():
    # 4 * block_q * block_kv * D per kept tile per query head: a per-head keep
    # counts each head's tiles once, a head-shared keep once per query head
    wl = workloads.get("gqa")
    keep = torch.zeros(wl.B, wl.Hq, wl.NQ, wl.NK, dtype=torch.int8)
    keep[0, 0, 0, :5] = 1
    keep[1, 3, 7, 2] = 1
    per_tile = 4 * 128 * 64 * 128
    assert bench.kept_tile_flops(keep, wl) == 6 * per_tile
    shared = torch.zeros(wl.B, 1, wl.NQ, wl.NK, dtype=torch.int8)
    shared[0, 0, 0, :5] = 1
    assert bench.kept_tile_flops(shared, wl) == 5 * wl.Hq * per_tile


def test_plan_kept_flops_by_hand():
    # tiny: 8 query tiles x 16 kv tiles, 2 diagonal tiles per row, 14
    # candidates, ceil(14 * 0.3) = 5, so 7 kept per row; 2 heads; D = 64
    wl = workloads.get("tiny")
    assert bench.plan_kept_flops(wl, None, None) == 7 * 8 * 2 * 4 * 128 * 64 * 64
    # head_shared: 53 kept per row of 256, one keep head for 32 query heads
    wl = workloads.get("head_shared")
    assert bench.plan_kept_flops(wl, None, None) == 53 * 256 * 32 * 4 * 128 * 64 * 128
    # gqa: 40 kept per row, 64 rows, 2 batches, 16 heads
    wl = workloads.get("gqa")
    assert bench.plan_kept_flops(wl, None, None) == 40 * 64 * 2 * 16 * 4 * 128 * 64 * 128


def test_oracle_units_cover_each_kv_group_once():
    assert bench.oracle_units(workloads.get("gqa")) == [(b, hk) for b in range(2) for hk in range(4)]
    assert bench.oracle_units(workloads.get("head_shared")) == [(0, None)]
