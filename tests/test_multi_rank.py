"""The bench's multi-rank host logic with world size 2 over gloo on the CPU:
process-group setup from the torchrun environment, barriers, max/sum over
ranks, independent per-rank batches (weak scaling, no data-path
collective), and the reference arm printing on rank 0 only."""
import io
import os
import socket
import contextlib

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    try:
        import bench
        import oracle
        import workloads
        r, w, local = bench.dist_setup("gloo")
        assert (r, w, local) == (rank, world, rank)
        cpu = torch.device("cpu")
        bench.barrier(w, cpu)
        # per-rank independent batch of the same workload
        wl = workloads.get("tiny")
        inp = workloads.make_inputs(wl, seed=bench.rank_seed(r))
        spec = oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
        keep = oracle.select_blocks(inp["q"].double().numpy(), inp["k"].double().numpy(), spec)
        flops = float(keep.sum()) * 4 * 128 * 64 * wl.D
        tot = bench.sum_over_ranks(flops, w, cpu)
        mx = bench.max_over_ranks(float(rank + 1), w, cpu)
        first = float(inp["q"][0, 0, 0, 0])
        firsts = [torch.zeros(1) for _ in range(w)]
        torch.distributed.all_gather(firsts, torch.tensor([first]))
        # reference arm: only rank 0 prints
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(bench_args())
        torch.distributed.destroy_process_group()
        q.put((rank, flops, tot, mx, [float(f) for f in firsts], buf.getvalue()))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e)))


def bench_args():
    import argparse
    return argparse.Namespace(workload="tiny", steps=1, warmup=3, cpu_seconds=1.0)


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        item = q.get(timeout=300)
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert res[r][1] != "error", res[r]
    f0, f1 = res[0][1], res[1][1]
    assert res[0][2] == pytest.approx(f0 + f1) and res[1][2] == pytest.approx(f0 + f1)
    assert res[0][3] == 2.0 and res[1][3] == 2.0
    # ranks draw different batches
    assert res[0][4][0] != res[0][4][1]
    # reference arm: one JSON line from rank 0, nothing from rank 1
    import json
    line = json.loads(res[0][5].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert res[1][5] == ""


# ---------------------------------------------------------------- one problem split over ranks

def test_rank_boxes_cover_every_unit_once():
    from top_kv_tile_b200 import shard
    for B in (1, 2, 3, 5):
        for Hkv in (1, 2, 3, 8):
            for world in (1, 2, 3, 4, 7):
                seen = []
                for r in range(world):
                    for box in shard.rank_boxes(B, Hkv, r, world):
                        assert box.b1 - box.b0 == 1 or (box.hk0, box.hk1) == (0, Hkv), box
                        seen += box.units()
                assert seen == shard.units(B, Hkv), (B, Hkv, world)


def _split_worker(rank, world, port, q):
    """Each rank runs the oracle's path on its own units of one problem; the
    results are gathered on every rank. Head-shared scoring gathers the
    pooled vectors of every head first (the one exchange the split needs)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    try:
        import bench
        import oracle
        import workloads
        from top_kv_tile_b200 import shard
        bench.dist_setup("gloo")
        results = {}
        for name in ("cross_small", "head_shared_small"):
            wl = workloads.get(name)
            inp = workloads.make_inputs(wl)
            qn, kn, vn = (inp[x].double().numpy() for x in "qkv")
            spec = oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
            g = wl.Hq // wl.Hkv
            outs = {}
            if wl.head_shared:
                assert wl.B == 1
                lo, hi = shard.head_range(wl.Hkv, rank, world)
                pq = oracle.pool_blocks(qn[:, lo * g:hi * g], wl.block_q)
                pk = oracle.pool_blocks(kn[:, lo:hi], wl.block_kv)
                counts_q = [(shard.head_range(wl.Hkv, r, world)[1] - shard.head_range(wl.Hkv, r, world)[0]) * g
                            for r in range(world)]
                counts_k = [c // g for c in counts_q]
                pq_all = shard.gather_heads(torch.from_numpy(pq), counts_q).numpy()
                pk_all = shard.gather_heads(torch.from_numpy(pk), counts_k).numpy()
                keep = oracle.select_pooled(pq_all, pk_all, spec, inp["pins"], inp["drops"])
                qs, ks, vs = qn[:, lo * g:hi * g], kn[:, lo:hi], vn[:, lo:hi]
                o, l = oracle.block_sparse_attention(qs, ks, vs, keep, wl.block_q, wl.block_kv, wl.scale)
                for hh in range(hi * g - lo * g):
                    outs[(0, lo * g + hh)] = (o[0, hh], l[0, hh])
                keeps = {"shared": keep}
            else:
                keeps = {}
                for box in shard.rank_boxes(wl.B, wl.Hkv, rank, world):
                    sl_q = (slice(box.b0, box.b1), slice(box.hk0 * g, box.hk1 * g))
                    sl_k = (slice(box.b0, box.b1), slice(box.hk0, box.hk1))
                    keep = oracle.select_blocks(qn[sl_q], kn[sl_k], spec, inp["pins"], inp["drops"])
                    o, l = oracle.block_sparse_attention(qn[sl_q], kn[sl_k], vn[sl_k], keep, wl.block_q,
                                                         wl.block_kv, wl.scale)
                    for bi, b in enumerate(range(box.b0, box.b1)):
                        for hi_, h in enumerate(range(box.hk0 * g, box.hk1 * g)):
                            outs[(b, h)] = (o[bi, hi_], l[bi, hi_])
                            keeps[(b, h)] = keep[bi, hi_]
            gathered = [None] * world
            torch.distributed.all_gather_object(gathered, (outs, keeps))
            results[name] = gathered
        torch.distributed.destroy_process_group()
        q.put((rank, results))
    except Exception as e:  # report instead of hanging the parent
        import traceback
        q.put((rank, "error", traceback.format_exc()))


def test_two_ranks_split_one_problem_match_one_rank():
    import oracle
    import workloads
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        item = q.get(timeout=300)
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert res[r][1] != "error", res[r][2]
    for name in ("cross_small", "head_shared_small"):
        wl = workloads.get(name)
        inp = workloads.make_inputs(wl)
        qn, kn, vn = (inp[x].double().numpy() for x in "qkv")
        spec = oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
        keep = oracle.select_blocks(qn, kn, spec, inp["pins"], inp["drops"])
        o, l = oracle.block_sparse_attention(qn, kn, vn, keep, wl.block_q, wl.block_kv, wl.scale)
        for r in range(2):
            parts = res[r][1][name]  # every rank gathered every rank's part
            union = {}
            for outs, keeps in parts:
                assert not (set(union) & set(outs)), "a unit was computed by two ranks"
                union.update(outs)
                for key, kr in keeps.items():
                    if key == "shared":
                        assert np.array_equal(kr, keep)  # the same keep on every rank
                    else:
                        assert np.array_equal(kr, keep[key[0], key[1]])
            assert set(union) == {(b, h) for b in range(wl.B) for h in range(wl.Hq)}
            for (b, h), (ob, lb) in union.items():
                assert np.array_equal(ob, o[b, h]) and np.array_equal(lb, l[b, h]), (name, b, h)
