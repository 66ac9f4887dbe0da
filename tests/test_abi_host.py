"""The C ABI on the host: the library builds for sm_100a, loads, exports every
entry point include/nsa.h declares, sizes workspaces, and rejects invalid
arguments before any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nsa():
    from top_kv_tile_b200 import build
    build.build()
    import top_kv_tile_b200
    return top_kv_tile_b200


def _declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "nsa.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_[a-z_0-9]+)\s*\(", hdr)))


def test_every_declared_symbol_is_exported(nsa):
    syms = _declared_symbols()
    assert "nsa_forward" in syms and "nsa_select" in syms and len(syms) >= 10
    lib = ctypes.CDLL(nsa.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), f"{s} declared in include/nsa.h but not exported"
    assert set(nsa.SYMBOLS) == set(syms)


def test_library_is_sm100a_only(nsa):
    assert "sm_100a" in nsa.nsa_version()


def _layout(B, Hq, Hkv, Sq, Skv, D, bq=128, bkv=64, hs=False):
    """Workspace bytes: the largest of nsa_forward's, nsa_select's and
    nsa_block_sparse_attn_fwd's layouts (each region 256-byte aligned)."""
    a = lambda x: (x + 255) // 256 * 256
    NQ, NK = -(-Sq // bq), -(-Skv // bkv)
    Hs = 1 if hs else Hq
    means = (a(B * NQ * D * 4) + a(B * NK * D * 4)) if hs else 0
    # flags, per-kv-group counters, pooled q, pooled k, head means, lists
    # tensor-core score scratch (B, Hs, NQ, NK rounded up to 128) float32
    # when the pooled keys of a head exceed 64 KB and the row has at most
    # 2048 tiles
    nkp = -(-NK // 128) * 128
    use_tc = NK * D * 4 > 64 * 1024 and nkp <= 2048
    tc = a(B * Hs * NQ * nkp * 4) if use_tc else 0
    # and the tf32 hi and lo parts of the scored keys (Hkv heads, or the
    # one head mean)
    split = 2 * a(B * (1 if hs else Hkv) * NK * D * 4) if use_tc else 0
    fwd = 256 + a(B * Hkv * 4) + a(B * Hq * NQ * D * 4) + a(B * Hkv * NK * D * 4) + means \
        + a(B * Hs * NQ * 4) + a(B * Hs * NQ * NK * 2) + tc + split
    sel = 256 + means + tc + split
    NQa, NKa = -(-Sq // 128), -(-Skv // 64)
    att = 256 + a(B * Hq * NQa * 4) + a(B * Hq * NQa * NKa * 2)
    return max(fwd, sel, att)


@pytest.mark.parametrize("dims,hs", [((2, 16, 4, 8192, 8192, 128), False),
                                     ((1, 32, 8, 32768, 32768, 128), True),
                                     ((4, 8, 8, 4096, 16000, 64), False),
                                     ((1, 2, 1, 100, 700, 64), False),
                                     ((1, 64, 8, 131072, 131072, 128), False)])
def test_workspace_bytes(nsa, dims, hs):
    spec = nsa.SparseSpec(0.3, 128, 64, hs, False)
    assert nsa.nsa_workspace_bytes(*dims, spec) == _layout(*dims, hs=hs)


def test_workspace_bytes_invalid(nsa):
    assert nsa.nsa_workspace_bytes(0, 1, 1, 1, 1, 64, nsa.SparseSpec()) == 0
    assert nsa.nsa_workspace_bytes(1, 1, 1, 1, 1, 64, nsa.SparseSpec(block_q=0)) == 0


def _status(nsa, st):
    return st, nsa.nsa_last_error()


def test_invalid_arguments_rejected_on_host(nsa):
    L = nsa.lib()
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: validation fails first
    spec = nsa.nsa_spec(0.3, 128, 64, 0, 0)
    # NULL input
    st = L.nsa_pool(None, 1, 1, 128, 64, 128, fake, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "NULL" in nsa.nsa_last_error()
    # unsupported head dim
    st = L.nsa_pool(fake, 1, 1, 128, 96, 128, fake, None)
    assert st == nsa.NSA_ERR_UNSUPPORTED and "96" in nsa.nsa_last_error()
    # misaligned pointer
    st = L.nsa_pool(P(0x10008), 1, 1, 128, 64, 128, fake, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "aligned" in nsa.nsa_last_error()
    # budget outside (0, 1]
    for bad in (0.0, -0.1, 1.5, float("nan")):
        s2 = nsa.nsa_spec(bad, 128, 64, 0, 0)
        st = L.nsa_forward(fake, fake, fake, 1, 2, 2, 1024, 1024, 64, ctypes.byref(s2), None, None, None, None,
                           0.125, fake, fake, None, P(0x10000), 1 << 30, None)
        assert st == nsa.NSA_ERR_INVALID_ARG and "budget" in nsa.nsa_last_error()
    # GQA head ratio
    st = L.nsa_forward(fake, fake, fake, 1, 3, 2, 1024, 1024, 64, ctypes.byref(spec), None, None, None, None,
                       0.125, fake, fake, None, P(0x10000), 1 << 30, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "multiple" in nsa.nsa_last_error()
    # attention tile geometry
    s3 = nsa.nsa_spec(0.3, 64, 64, 0, 0)
    st = L.nsa_forward(fake, fake, fake, 1, 2, 2, 1024, 1024, 64, ctypes.byref(s3), None, None, None, None,
                       0.125, fake, fake, None, P(0x10000), 1 << 30, None)
    assert st == nsa.NSA_ERR_UNSUPPORTED and "block_q=128" in nsa.nsa_last_error()
    # workspace too small
    st = L.nsa_forward(fake, fake, fake, 1, 2, 2, 1024, 1024, 64, ctypes.byref(spec), None, None, None, None,
                       0.125, fake, fake, None, P(0x10000), 1024, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "workspace" in nsa.nsa_last_error()
    # pins without strides
    st = L.nsa_forward(fake, fake, fake, 1, 2, 2, 1024, 1024, 64, ctypes.byref(spec), fake, None, None, None,
                       0.125, fake, fake, None, P(0x10000), 1 << 30, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "strides" in nsa.nsa_last_error()
    # non-finite scale
    st = L.nsa_block_sparse_attn_fwd(fake, fake, fake, 1, 2, 2, 1024, 1024, 64, None, 1, 128, 64,
                                     float("inf"), fake, fake, None, 0, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "scale" in nsa.nsa_last_error()
    # NULL spec
    st = L.nsa_select(fake, fake, 1, 2, 2, 8, 16, 64, None, None, None, None, None, fake, fake, fake,
                      ctypes.byref(ctypes.c_int()), fake, 256, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "spec" in nsa.nsa_last_error()
    # key mask: negative strides, strides without a mask
    neg = (ctypes.c_int64 * 3)(2048, -1024, 1)
    st = L.nsa_block_sparse_attn_fwd_masked(fake, fake, fake, 1, 2, 2, 1024, 1024, 64, None, 1, 128, 64,
                                            fake, neg, 0.125, fake, fake, None, 0, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "strides" in nsa.nsa_last_error()
    ok = (ctypes.c_int64 * 3)(2048, 1024, 1)
    st = L.nsa_block_sparse_attn_fwd_masked(fake, fake, fake, 1, 2, 2, 1024, 1024, 64, None, 1, 128, 64,
                                            None, ok, 0.125, fake, fake, None, 0, None)
    assert st == nsa.NSA_ERR_INVALID_ARG and "key mask" in nsa.nsa_last_error()


def test_empty_and_oversized_inputs_rejected_on_host(nsa):
    # empty inputs (a zero size) and sizes past the documented maxima are
    # refused before anything is enqueued
    L = nsa._lib
    P = ctypes.c_void_p
    fake = P(0x10000)
    spec = nsa.SparseSpec(0.3, 128, 64, False, False).c()
    for dims in ((0, 2, 2, 1024, 1024, 64), (1, 2, 2, 0, 1024, 64), (1, 2, 2, 1024, 0, 64), (1, 0, 1, 1024, 1024, 64)):
        st = L.nsa_forward(fake, fake, fake, *dims, ctypes.byref(spec), None, None, None, None, 0.125, fake, fake,
                           None, fake, 1 << 30, None)
        assert st == nsa.NSA_ERR_INVALID_ARG and "positive" in nsa.nsa_last_error(), dims
        st = L.nsa_block_sparse_attn_fwd(fake, fake, fake, *dims, None, 1, 128, 64, 0.125, fake, fake, None, 0,
                                         None)
        assert st == nsa.NSA_ERR_INVALID_ARG, dims
    st = L.nsa_pool(fake, 1, 1, 0, 64, 128, fake, None)
    assert st == nsa.NSA_ERR_INVALID_ARG
    # more kv tiles than the 16-bit kept lists index (65535)
    st = L.nsa_block_sparse_attn_fwd(fake, fake, fake, 1, 1, 1, 128, 64 * 65536, 64, None, 1, 128, 64, 0.125,
                                     fake, fake, None, 0, None)
    assert st == nsa.NSA_ERR_UNSUPPORTED and "65535" in nsa.nsa_last_error()
    # more query tiles than the backward's 16-bit query lists index
    st = L.nsa_block_sparse_attn_bwd(fake, fake, fake, fake, fake, fake, 1, 1, 1, 128 * 65536, 64, 64, None, 1,
                                     128, 64, 0.125, fake, fake, fake, P(0x100000), 1 << 40, None)
    assert st == nsa.NSA_ERR_UNSUPPORTED and "65535" in nsa.nsa_last_error()


def test_package_submodules_import_without_the_library():
    # ``from top_kv_tile_b200 import build`` must reach the build module even
    # when libnsa.so is missing or stale (a fresh checkout builds it)
    import top_kv_tile_b200
    with pytest.raises(AttributeError):
        top_kv_tile_b200.__getattr__("build")


def test_python_binding_rejects_cpu_tensors(nsa):
    import torch
    x = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        nsa.nsa_pool(x, 128)


def test_wrappers_with_a_stream_allocate_on_it():
    # every binding call that takes a `stream` runs under it, so the tensors
    # it allocates belong to the stream its kernels are enqueued on
    import inspect
    from top_kv_tile_b200 import binding
    seen = []
    for name in dir(binding):
        f = getattr(binding, name)
        if inspect.isfunction(f) and name.startswith("nsa_"):
            if "stream" in inspect.signature(inspect.unwrap(f)).parameters:
                assert getattr(f, "__wrapped__", None) is not None, name
                seen.append(name)
    assert "nsa_forward" in seen and "nsa_block_sparse_attn_bwd" in seen and len(seen) >= 10


def test_stream_given_by_position_is_entered(monkeypatch):
    # a stream passed positionally must be entered like one passed by keyword,
    # or the wrapper's allocations would land on the current stream instead
    from top_kv_tile_b200 import binding
    entered = []

    class Ctx:
        def __init__(self, s):
            self.s = s

        def __enter__(self):
            entered.append(self.s)

        def __exit__(self, *exc):
            return False

    monkeypatch.setattr(binding.torch.cuda, "stream", Ctx)

    @binding._on_caller_stream
    def f(x, block, out=None, stream=None):
        return stream

    s = object()
    assert f(1, 2, None, s) is s and entered == [s]
    assert f(1, 2, stream=s) is s and entered == [s, s]
    assert f(1, 2) is None and entered == [s, s]


def test_selftest_timeout_and_launch_count_on_host(nsa):
    L = nsa.lib()
    # invalid arguments are rejected before any CUDA call
    assert L.nsa_selftest_timeout(2, 1000, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_selftest_timeout(0, 0, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_selftest_timeout(1, 1 << 40, None) == nsa.NSA_ERR_INVALID_ARG
    assert "limit_cycles" in nsa.nsa_last_error()
    # the launch counter is a plain host read
    n = nsa.nsa_kernel_launches()
    assert isinstance(n, int) and n >= 0 and nsa.nsa_kernel_launches() == n
