"""nsa_forward_noalloc: the whole path for callers that may not allocate
device memory (their memory belongs to another allocator, or cudaMalloc's
implicit synchronisation is not allowed where they run). The call takes no
workspace: its scratch is the library's fixed device array. Checked through
the C ABI against nsa_forward with a caller workspace, on consecutive calls
that share the array. Collected last so a stop-at-first-failure run has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from top_kv_tile_b200 import build
    build.build()
    import top_kv_tile_b200
    assert torch.cuda.is_available()
    return top_kv_tile_b200


def _inputs(name, seed=0):
    wl = workloads.get(name)
    inp = workloads.make_inputs(wl, seed=seed)
    d = {x: inp[x].cuda() for x in "qkv"}
    for m in ("pins", "drops"):
        d[m] = None if inp[m] is None else torch.from_numpy(inp[m]).cuda()
    return wl, d


def _mask_args(m):
    if m is None:
        return None, None
    st = [0 if m.shape[i] == 1 else m.stride(i) for i in range(4)]
    return ctypes.c_void_p(m.data_ptr()), (ctypes.c_int64 * 4)(*st)


def _noalloc_c_abi(nsa, wl, d):
    """One nsa_forward_noalloc call straight through the C ABI."""
    out = torch.empty_like(d["q"])
    lse = torch.empty(wl.B, wl.Hq, wl.Sq, dtype=torch.float32, device="cuda")
    keep = torch.empty(wl.B, wl.Hs, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    spec = nsa.nsa_spec(wl.budget, wl.block_q, wl.block_kv, int(wl.head_shared), int(wl.force))
    pm, ps = _mask_args(d["pins"])
    dm, ds = _mask_args(d["drops"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = nsa.lib().nsa_forward_noalloc(
        ctypes.c_void_p(d["q"].data_ptr()), ctypes.c_void_p(d["k"].data_ptr()), ctypes.c_void_p(d["v"].data_ptr()),
        wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Skv, wl.D, ctypes.byref(spec), pm, ps, dm, ds, ctypes.c_float(wl.scale),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(keep.data_ptr()), stream)
    assert st == nsa.NSA_OK, nsa.nsa_last_error()
    torch.cuda.synchronize()
    return out, lse, keep


def _with_workspace(nsa, wl, d):
    keep = torch.empty(wl.B, wl.Hs, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    spec = nsa.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    out, lse = nsa.nsa_forward(d["q"], d["k"], d["v"], spec, wl.scale, d["pins"], d["drops"], keep_out=keep)
    torch.cuda.synchronize()
    return out, lse, keep


def _same(a, b):
    out, lse, keep = a
    ro, rl, rk = b
    assert torch.equal(keep, rk)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(),
                           ro.float().cpu().numpy().astype(np.float64), rl.cpu().numpy().astype(np.float64))


def test_noalloc_matches_workspace_path_on_consecutive_calls(nsa):
    # the paths a call can take: the single cooperative select kernel
    # (gqa_small, cross_small), pooling first with the head means
    # (head_shared_small), tensor-core scores for long rows (long_kv_hs) and
    # a partial last tile on both axes (ragged)
    names = ["gqa_small", "cross_small", "head_shared_small", "long_kv_hs", "ragged"]
    cases = [_inputs(n) for n in names]
    for wl, _ in cases:
        spec = nsa.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
        assert nsa.nsa_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Skv, wl.D, spec) <= nsa.NOALLOC_SCRATCH_BYTES
    refs = [_with_workspace(nsa, wl, d) for wl, d in cases]
    # two calls in a row per case, interleaved so each call finds another
    # path's leftovers in the shared scratch array
    for _ in range(2):
        for (wl, d), ref in zip(cases, refs):
            _same(_noalloc_c_abi(nsa, wl, d), ref)
    nsa.nsa_device_status()


def test_noalloc_rejects_sizes_above_the_array(nsa):
    wl = workloads.get("large2d")
    spec = nsa.nsa_spec(wl.budget, wl.block_q, wl.block_kv, 0, 0)
    fake = ctypes.c_void_p(0x10000)  # rejected on the host before any use
    st = nsa.lib().nsa_forward_noalloc(fake, fake, fake, wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Skv, wl.D,
                                       ctypes.byref(spec), None, None, None, None, ctypes.c_float(wl.scale),
                                       fake, fake, None, None)
    assert st == nsa.NSA_ERR_INVALID_ARG
    msg = nsa.nsa_last_error()
    assert "scratch" in msg and str(nsa.NOALLOC_SCRATCH_BYTES) in msg
