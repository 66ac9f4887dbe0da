"""Backward over kept tiles: nsa_block_sparse_attn_bwd (dQ, dK, dV) against
the oracle's block_sparse_attention_bwd on the same seeded inputs, keep and
upstream gradient; the forward that feeds it is the library's own."""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

CASES = ["tiny", "gqa_small", "head_shared_small", "cross_small", "ragged", "ragged_cross", "nq1",
         "dense_force", "large2d_small", "long_kv_ragged", "long_kv_2k"]


@pytest.fixture(scope="module")
def nsa():
    from top_kv_tile_b200 import build
    build.build()
    import top_kv_tile_b200
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return top_kv_tile_b200


@functools.lru_cache(maxsize=None)
def _case(name):
    wl = workloads.get(name)
    inp = workloads.make_inputs(wl)
    q, k, _ = (inp[x].double().numpy() for x in "qkv")
    spec = oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    keep = oracle.select_blocks(q, k, spec, inp["pins"], inp["drops"])
    dout = workloads.upstream_grad(wl)
    return wl, inp, keep, dout


def _oracle_fwd(inp, keep, scale):
    """The forward's outputs as the backward receives them, from the oracle:
    O rounded to bf16 (the forward stores O in bf16) and LSE in f32."""
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    O, L = oracle.block_sparse_attention(q, k, v, keep, 128, 64, scale)
    return torch.from_numpy(O).to(torch.bfloat16), torch.from_numpy(L).float()


def _gpu_bwd(nsa, wl, inp, keep, dout, out, lse):
    q, k, v = (inp[x].cuda() for x in "qkv")
    kt = None if keep is None else torch.from_numpy(keep).cuda()
    dq, dk, dv = nsa.nsa_block_sparse_attn_bwd(q, k, v, out.cuda(), lse.cuda(), dout.cuda(), kt, wl.scale)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    return [t.float().cpu().numpy() for t in (dq, dk, dv)]


def _check_bwd(nsa, wl, inp, keep, dout):
    # the backward as a function of its inputs: the same q, k, v, keep,
    # stored O, LSE and dO on both sides
    out, lse = _oracle_fwd(inp, keep, wl.scale)
    got = _gpu_bwd(nsa, wl, inp, keep, dout, out, lse)
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    ref = oracle.block_sparse_attention_bwd(q, k, v, keep, 128, 64, wl.scale, dout.double().numpy(),
                                            out=out.double().numpy())
    for g, r, n in zip(got, ref, ("dq", "dk", "dv")):
        parity.check_grad(g, r, n)
    return got


@pytest.mark.parametrize("name", CASES)
def test_backward_matches_oracle(nsa, name):
    wl, inp, keep, dout = _case(name)
    _check_bwd(nsa, wl, inp, keep, dout)


def test_backward_dense_keep_none(nsa):
    wl, inp, _, dout = _case("ragged")
    _check_bwd(nsa, wl, inp, None, dout)


@pytest.mark.parametrize("name", ["gqa_small", "head_shared_small", "ragged_cross"])
def test_forward_then_backward_against_the_exact_gradient(nsa, name):
    # the library's forward feeding its backward, against the exact gradient
    # (Dv from the exact O); on these workloads no row's softmax is peaked
    # enough for the bf16 rounding of the stored O to matter
    wl, inp, keep, dout = _case(name)
    q, k, v = (inp[x].cuda() for x in "qkv")
    kt = torch.from_numpy(keep).cuda()
    out, lse = nsa.nsa_block_sparse_attn_fwd(q, k, v, kt, wl.scale)
    got = _gpu_bwd(nsa, wl, inp, keep, dout, out, lse)
    qn, kn, vn = (inp[x].double().numpy() for x in "qkv")
    ref = oracle.block_sparse_attention_bwd(qn, kn, vn, keep, 128, 64, wl.scale, dout.double().numpy())
    for g, r, n in zip(got, ref, ("dq", "dk", "dv")):
        parity.check_grad(g, r, n)


def test_backward_empty_rows_and_unkept_tiles(nsa):
    # a keep with a whole row empty and a kv tile no row keeps: dq of the row
    # and dk, dv of the tile are exactly 0
    wl, inp, keep, dout = _case("gqa_small")
    keep = keep.copy()
    keep[0, 1, 3] = 0
    keep[0, :, :, 5] = 0
    got = _check_bwd(nsa, wl, inp, keep, dout)
    assert np.all(got[0][0, 1, 384:512] == 0)
    assert np.all(got[1][0, :, 320:384] == 0) and np.all(got[2][0, :, 320:384] == 0)


def test_backward_full_size_gqa_sampled(nsa):
    # the GQA workload at full size, the library's own selection and forward
    # feeding its backward; sampled dQ tile rows and sampled dK/dV kv tiles
    # against the exact gradient, recomputed by the oracle on the rows that
    # determine them (a dQ row depends on its own keep row; a kv tile's dK/dV
    # on the rows that kept it)
    wl = workloads.get("gqa")
    inp = workloads.make_inputs(wl)
    q, k, v = (inp[x].cuda() for x in "qkv")
    spec = nsa.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    keep = torch.empty(wl.B, wl.Hs, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    out, lse = nsa.nsa_forward(q, k, v, spec, wl.scale, keep_out=keep)
    dout = workloads.upstream_grad(wl)
    dq, dk, dv = nsa.nsa_block_sparse_attn_bwd(q, k, v, out, lse, dout.cuda(), keep, wl.scale)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    gk = keep.cpu().numpy()
    qn, kn, vn = (inp[x].double().numpy() for x in "qkv")
    don = dout.double().numpy()
    g = wl.Hq // wl.Hkv
    rng = np.random.default_rng(99)
    for _ in range(4):
        b, h, i = int(rng.integers(wl.B)), int(rng.integers(wl.Hq)), int(rng.integers(wl.NQ))
        hk = h // g
        rows = slice(i * 128, (i + 1) * 128)
        sq, sk, sv = qn[b:b + 1, h:h + 1, rows], kn[b:b + 1, hk:hk + 1], vn[b:b + 1, hk:hk + 1]
        skeep = gk[b:b + 1, h:h + 1, i:i + 1]
        rq, _, _ = oracle.block_sparse_attention_bwd(sq, sk, sv, skeep, 128, 64, wl.scale,
                                                     don[b:b + 1, h:h + 1, rows])
        parity.check_grad(dq[b, h, rows].float().cpu().numpy(), rq[0, 0], "dq")
    for _ in range(3):
        b, hk, j = int(rng.integers(wl.B)), int(rng.integers(wl.Hkv)), int(rng.integers(wl.NK))
        rk = np.zeros((64, wl.D))
        rv = np.zeros((64, wl.D))
        for h in range(hk * g, (hk + 1) * g):
            tiles = np.nonzero(gk[b, h, :, j])[0]
            if len(tiles) == 0:
                continue
            idx = np.concatenate([np.arange(t * 128, (t + 1) * 128) for t in tiles])
            sq, sk, sv = qn[b:b + 1, h:h + 1, idx], kn[b:b + 1, hk:hk + 1], vn[b:b + 1, hk:hk + 1]
            skeep = gk[b:b + 1, h:h + 1, tiles]
            _, ek, ev = oracle.block_sparse_attention_bwd(sq, sk, sv, skeep, 128, 64, wl.scale,
                                                          don[b:b + 1, h:h + 1, idx])
            rk += ek[0, 0, j * 64:(j + 1) * 64]
            rv += ev[0, 0, j * 64:(j + 1) * 64]
        parity.check_grad(dk[b, hk, j * 64:(j + 1) * 64].float().cpu().numpy(), rk, "dk")
        parity.check_grad(dv[b, hk, j * 64:(j + 1) * 64].float().cpu().numpy(), rv, "dv")


MASK_CASES = [("tiny", "random50", True), ("gqa_small", "padding", True), ("ragged_cross", "head0_off", True),
              ("large2d_small", "random50", False), ("ragged", "prefix_off", True)]


@pytest.mark.parametrize("name,kind,per_head", MASK_CASES)
def test_masked_backward_matches_oracle(nsa, name, kind, per_head):
    # the key-masked forward's gradients: stored O (bf16) and LSE from the
    # oracle's masked forward on both sides
    wl, inp, keep, dout = _case(name)
    km = np.broadcast_to(workloads.key_mask(wl, kind, per_head=per_head), (wl.B, wl.Hkv, wl.Skv))
    q, k, v = (inp[x].double().numpy() for x in "qkv")
    O, L = oracle.block_sparse_attention(q, k, v, keep, 128, 64, wl.scale, km)
    out = torch.from_numpy(O).to(torch.bfloat16)
    lse = torch.from_numpy(L).float()
    qd, kd, vd = (inp[x].cuda() for x in "qkv")
    kt = torch.from_numpy(keep).cuda()
    kmt = torch.from_numpy(np.ascontiguousarray(workloads.key_mask(wl, kind, per_head=per_head))).cuda()
    got = nsa.nsa_block_sparse_attn_bwd(qd, kd, vd, out.cuda(), lse.cuda(), dout.cuda(), kt, wl.scale, kmask=kmt)
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    ref = oracle.block_sparse_attention_bwd(q, k, v, keep, 128, 64, wl.scale, dout.double().numpy(), km,
                                            out=out.double().numpy())
    for g, r, n in zip(got, ref, ("dq", "dk", "dv")):
        parity.check_grad(g.float().cpu().numpy(), r, n)
    # masked key rows get no gradient
    gk = got[1].float().cpu().numpy()
    gv = got[2].float().cpu().numpy()
    assert np.all(gk[~km] == 0) and np.all(gv[~km] == 0)


def test_all_true_mask_backward_is_bit_identical(nsa):
    wl, inp, keep, dout = _case("gqa_small")
    out, lse = _oracle_fwd(inp, keep, wl.scale)
    qd, kd, vd = (inp[x].cuda() for x in "qkv")
    kt = torch.from_numpy(keep).cuda()
    a = nsa.nsa_block_sparse_attn_bwd(qd, kd, vd, out.cuda(), lse.cuda(), dout.cuda(), kt, wl.scale)
    ones = torch.ones(wl.B, wl.Hkv, wl.Skv, dtype=torch.int8, device="cuda")
    b = nsa.nsa_block_sparse_attn_bwd(qd, kd, vd, out.cuda(), lse.cuda(), dout.cuda(), kt, wl.scale, kmask=ones)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
