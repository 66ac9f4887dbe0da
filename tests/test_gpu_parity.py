"""GPU parity: the CUDA path through the C ABI against the CPU oracle, on the
same seeded inputs (workloads/). Sizes span several tiles and ragged tails;
the oracle finishes each in seconds."""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "gqa_small", "head_shared_small", "cross_small", "large2d_small",
         "ragged", "ragged_cross", "nq1", "dense_force", "long_kv_small", "long_kv_ragged", "long_kv_hs", "long_kv_2k",
         "long_kv_4k", "long_kv_8k_hs"]


@pytest.fixture(scope="module")
def nsa():
    from top_kv_tile_b200 import build
    build.build()
    import top_kv_tile_b200
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return top_kv_tile_b200


def _spec_o(wl):
    return oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)


def _spec_g(nsa, wl):
    return nsa.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)


@functools.lru_cache(maxsize=None)
def _case(name):
    wl = workloads.get(name)
    inp = workloads.make_inputs(wl)
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    keep, scores, plan = oracle.select_blocks(q, k, _spec_o(wl), inp["pins"], inp["drops"], return_scores=True)
    return wl, inp, keep, scores, plan


@functools.lru_cache(maxsize=None)
def _oracle_attn(name):
    wl, inp, keep, _, _ = _case(name)
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    return oracle.block_sparse_attention(q, k, v, keep, wl.block_q, wl.block_kv, wl.scale)


def _dev(inp):
    d = {x: inp[x].cuda() for x in "qkv"}
    for m in ("pins", "drops"):
        d[m] = None if inp[m] is None else torch.from_numpy(inp[m]).cuda()
    return d


@pytest.mark.parametrize("name", SMALL)
def test_pool(nsa, name):
    wl, inp, *_ = _case(name)
    d = _dev(inp)
    for x, blk in (("q", wl.block_q), ("k", wl.block_kv)):
        got = nsa.nsa_pool(d[x], blk).cpu().numpy().astype(np.float64)
        ref = oracle.pool_blocks(inp[x].double().numpy(), blk)
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("name", ["tiny", "gqa_small", "head_shared_small", "ragged"])
def test_score(nsa, name):
    wl, inp, _, scores, _ = _case(name)
    d = _dev(inp)
    pq = nsa.nsa_pool(d["q"], wl.block_q)
    pk = nsa.nsa_pool(d["k"], wl.block_kv)
    got = nsa.nsa_score(pq, pk, wl.head_shared).cpu().numpy().astype(np.float64)
    scale = np.abs(scores).max(axis=-1, keepdims=True)
    assert got.shape == scores.shape
    assert np.all(np.abs(got - scores) <= 1e-5 * scale + 1e-7)


@pytest.mark.parametrize("name", SMALL)
def test_select(nsa, name):
    wl, inp, keep, scores, plan = _case(name)
    d = _dev(inp)
    pq = nsa.nsa_pool(d["q"], wl.block_q)
    pk = nsa.nsa_pool(d["k"], wl.block_kv)
    gk, cnt, idx, dense = nsa.nsa_select(pq, pk, _spec_g(nsa, wl), d["pins"], d["drops"])
    assert dense is False
    gk = gk.cpu().numpy()
    stats = parity.check_keep_rows(gk, keep, scores, plan)
    assert stats["exact"] >= 0.95 * stats["rows"], stats
    parity.check_lists(gk, cnt.cpu().numpy(), idx.cpu().numpy())


@pytest.mark.parametrize("name", ["tiny", "cross_small", "ragged_cross"])
def test_keep_to_index(nsa, name):
    wl, inp, keep, *_ = _case(name)
    kt = torch.from_numpy(keep).cuda()
    cnt, idx = nsa.nsa_keep_to_index(kt)
    parity.check_lists(keep, cnt.cpu().numpy(), idx.cpu().numpy())


@pytest.mark.parametrize("name", SMALL)
def test_attention_from_oracle_keep(nsa, name):
    wl, inp, keep, *_ = _case(name)
    d = _dev(inp)
    kt = torch.from_numpy(keep).cuda()
    out, lse = nsa.nsa_block_sparse_attn_fwd(d["q"], d["k"], d["v"], kt, wl.scale)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    ro, rl = _oracle_attn(name)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)


@pytest.mark.parametrize("name", SMALL)
def test_forward_end_to_end(nsa, name):
    wl, inp, keep, scores, plan = _case(name)
    d = _dev(inp)
    keep_out = torch.empty(keep.shape, dtype=torch.int8, device="cuda")
    out, lse = nsa.nsa_forward(d["q"], d["k"], d["v"], _spec_g(nsa, wl), wl.scale, d["pins"], d["drops"],
                               keep_out=keep_out)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    gk = keep_out.cpu().numpy()
    parity.check_keep_rows(gk, keep, scores, plan)
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    if np.array_equal(gk, keep):
        ro, rl = _oracle_attn(name)
    else:
        ro, rl = oracle.block_sparse_attention(q, k, v, gk, wl.block_q, wl.block_kv, wl.scale)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)


def test_dense_short_circuit(nsa):
    # budget 1.0 with force off: the plan covers every candidate, the page
    # returns None (attend densely, drops not applied)
    wl = workloads.get("cross_small").with_(budget=1.0, force=False)
    inp = workloads.make_inputs(wl)
    d = _dev(inp)
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    assert oracle.select_blocks(q, k, _spec_o(wl), inp["pins"], inp["drops"]) is None
    pq = nsa.nsa_pool(d["q"], wl.block_q)
    pk = nsa.nsa_pool(d["k"], wl.block_kv)
    _, _, _, dense = nsa.nsa_select(pq, pk, _spec_g(nsa, wl), d["pins"], d["drops"])
    assert dense is True
    out, lse = nsa.nsa_forward(d["q"], d["k"], d["v"], _spec_g(nsa, wl), wl.scale, d["pins"], d["drops"])
    ro, rl = oracle.block_sparse_attention(q, k, v, None, wl.block_q, wl.block_kv, wl.scale)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)


def test_dense_attention_keep_none(nsa):
    wl = workloads.get("ragged")
    inp = workloads.make_inputs(wl)
    d = _dev(inp)
    out, lse = nsa.nsa_block_sparse_attn_fwd(d["q"], d["k"], d["v"], None, wl.scale)
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    ro, rl = oracle.block_sparse_attention(q, k, v, None, 128, 64, wl.scale)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)


def test_empty_rows_give_zero_and_neg_inf(nsa):
    # drops that forbid every tile of some rows (diagonal included)
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl)
    d = _dev(inp)
    drops = np.zeros((1, 1, wl.NQ, wl.NK), np.int8)
    drops[..., 3, :] = 1
    drops[..., 5, 10:] = 1
    keep_out = torch.empty(1, 2, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    out, lse = nsa.nsa_forward(d["q"], d["k"], d["v"], _spec_g(nsa, wl), wl.scale, None,
                               torch.from_numpy(drops).cuda(), keep_out=keep_out)
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    keep, scores, plan = oracle.select_blocks(q, k, _spec_o(wl), None, drops, return_scores=True)
    assert keep[0, :, 3].sum() == 0
    parity.check_keep_rows(keep_out.cpu().numpy(), keep, scores, plan)
    ro, rl = oracle.block_sparse_attention(q, k, v, keep, 128, 64, wl.scale)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)
    assert torch.all(out[:, :, 384:512] == 0)


@pytest.mark.parametrize("m", [-2, 3])
def test_keep_invariant_to_power_of_two_scaling(nsa, m):
    wl = workloads.get("gqa_small")
    inp = workloads.make_inputs(wl)
    d = _dev(inp)
    spec = _spec_g(nsa, wl)
    k0 = torch.empty(1, wl.Hq, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    k1 = torch.empty_like(k0)
    nsa.nsa_forward(d["q"], d["k"], d["v"], spec, keep_out=k0)
    nsa.nsa_forward((d["q"].float() * 2.0 ** m).bfloat16(), d["k"], d["v"], spec, keep_out=k1)
    assert torch.equal(k0, k1)


def test_budget_one_force_keeps_all_but_forbidden(nsa):
    wl = workloads.get("cross_small").with_(budget=1.0, force=True)
    inp = workloads.make_inputs(wl)
    d = _dev(inp)
    keep_out = torch.empty(wl.B, wl.Hq, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    nsa.nsa_forward(d["q"], d["k"], d["v"], _spec_g(nsa, wl), wl.scale, d["pins"], d["drops"], keep_out=keep_out)
    expect = np.broadcast_to(1 - inp["drops"], keep_out.shape)
    assert np.array_equal(keep_out.cpu().numpy(), expect)


def test_all_equal_scores_keep_lowest_indices(nsa):
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl)
    d = _dev(inp)
    q = torch.zeros_like(d["q"])
    keep_out = torch.empty(1, 2, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    nsa.nsa_forward(q, d["k"], d["v"], _spec_g(nsa, wl), wl.scale, keep_out=keep_out)
    ref = oracle.select_blocks(np.zeros(inp["q"].shape), inp["k"].double().numpy(), _spec_o(wl))
    assert np.array_equal(keep_out.cpu().numpy(), ref)


def test_device_status_clean(nsa):
    torch.cuda.synchronize()
    nsa.nsa_device_status()


@pytest.mark.parametrize("name,seed", [("long_kv_small", 0), ("long_kv_ragged", 0), ("gqa_small", 1)])
def test_tensor_core_scores_within_split_precision_bound(nsa, name, seed):
    # the 3xTF32 scores against the float64 scores of the same pooled
    # vectors: the dropped lo.lo term and the tf32 roundings leave about
    # 2^-21 of |q_d k_d| per product and the f32 accumulation over D terms
    # adds a few 2^-24 of sum_d |q_d k_d|; bound: 2^-18 of sum_d |q_d k_d|
    wl = workloads.get(name)
    g = torch.Generator().manual_seed(seed)
    pq = torch.randn(wl.B, wl.Hq, wl.NQ, wl.D, generator=g) * 3.0
    pk = torch.randn(wl.B, wl.Hkv, wl.NK, wl.D, generator=g) * 0.5
    got = nsa.nsa_score_tc(pq.cuda(), pk.cuda()).cpu().double().numpy()
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    q = pq.double().numpy()
    k = np.repeat(pk.double().numpy(), wl.Hq // wl.Hkv, axis=1)
    ref = np.einsum("bhid,bhjd->bhij", q, k)
    mag = np.einsum("bhid,bhjd->bhij", np.abs(q), np.abs(k))
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -18 * mag + 1e-30), float((err / mag).max())
    # far below the 2^-11 relative error of a single tf32 product
    assert (err / mag).max() < 2.0 ** -19


def _pair_keep_patterns(wl, seed):
    """Keep tensors whose neighbouring heads keep very different tiles: long
    runs kept by one head only, one head keeping nothing, identical lists,
    and independent random lists (rows cycle through the patterns)."""
    rng = np.random.default_rng(seed)
    keep = np.zeros((wl.B, wl.Hs, wl.NQ, wl.NK), dtype=np.int8)
    nk = wl.NK
    for b in range(wl.B):
        for hp in range(0, wl.Hq, 2):
            for i in range(wl.NQ):
                kind = (b * wl.Hq + hp + i) % 5
                a0 = np.zeros(nk, dtype=bool)
                a1 = np.zeros(nk, dtype=bool)
                if kind == 0:    # runs of 1..17 tiles alternating between the heads
                    j, cur = 0, 0
                    while j < nk:
                        r = int(rng.integers(1, 18))
                        (a0 if cur == 0 else a1)[j:j + r] = True
                        j += r
                        cur ^= 1
                elif kind == 1:  # head 0 keeps the first and last tiles, head 1 all between
                    a0[0] = a0[nk - 1] = True
                    a1[1:nk - 1] = True
                elif kind == 2:  # one head keeps nothing
                    a1[rng.random(nk) < 0.4] = True
                elif kind == 3:  # identical lists
                    a0[rng.random(nk) < 0.3] = True
                    a1[:] = a0
                else:            # independent
                    a0[rng.random(nk) < 0.2] = True
                    a1[rng.random(nk) < 0.5] = True
                keep[b, hp, i] = a0
                keep[b, hp + 1, i] = a1
    return keep


@pytest.mark.parametrize("name", ["long_kv_small", "long_kv_ragged"])
def test_attention_keep_patterns(nsa, name):
    # hand-made keep rows: long runs, empty rows, identical and independent
    # lists for the heads of a kv group, rows keeping nearly every tile
    wl = workloads.get(name)
    assert (wl.Hq // wl.Hkv) % 2 == 0 and not wl.head_shared
    inp = workloads.make_inputs(wl)
    d = _dev(inp)
    keep = _pair_keep_patterns(wl, seed=7)
    out, lse = nsa.nsa_block_sparse_attn_fwd(d["q"], d["k"], d["v"], torch.from_numpy(keep).cuda(), wl.scale)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    ro, rl = oracle.block_sparse_attention(q, k, v, keep, wl.block_q, wl.block_kv, wl.scale)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)


def test_attention_kv_index_beyond_int16(nsa):
    # kept-tile indices on both sides of 2^15 (the lists are uint16) and the
    # partial last tile of a 33,001-tile key axis; one row keeps nothing,
    # one keeps 300 tiles, and the last query tile is partial
    B, Hq, Hkv, D = 1, 2, 1, 64
    Sq, NK = 3 * 128 - 57, 33001
    Skv = (NK - 1) * 64 + 17
    gen = torch.Generator().manual_seed(5)
    q = torch.randn(B, Hq, Sq, D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Skv, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Skv, D, generator=gen).to(torch.bfloat16)
    NQ = (Sq + 127) // 128
    keep = np.zeros((B, Hq, NQ, NK), dtype=np.int8)
    rng = np.random.default_rng(9)
    fixed = [0, 1, 8191, 8192, 16384, 32766, 32767, 32768, 32769, NK - 2, NK - 1]
    keep[0, 0, 0, fixed] = 1
    keep[0, 0, 1, rng.choice(NK, 300, replace=False)] = 1
    keep[0, 0, 2, 32768:32768 + 40] = 1
    keep[0, 1, 0, rng.choice(np.arange(32000, NK), 25, replace=False)] = 1
    keep[0, 1, 2, [5, NK - 1]] = 1  # row (1, 1) keeps nothing
    out, lse = nsa.nsa_block_sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(keep).cuda(), D ** -0.5)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    ro, rl = oracle.block_sparse_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), keep, 128, 64,
                                           D ** -0.5)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)
