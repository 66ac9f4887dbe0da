"""Python binding of libnsa, the B200 library for fixed-budget block-sparse
attention (block selection as in automatic/modules/attention/sparse/selector.py,
followed by attention over the kept tiles).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, checks dtypes and shapes, and passes raw pointers and the
current CUDA stream to the C ABI declared in include/nsa.h. Every step of the
computation runs in the library's CUDA kernels. There is no CPU fallback: if
libnsa.so is missing or fails to load, importing this package raises.
"""
from __future__ import annotations

import ctypes
import functools
import inspect
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libnsa.so not found at {LIB_PATH}; build it with `python -m top_kv_tile_b200.build` "
        "(nvcc for sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

NSA_OK, NSA_ERR_INVALID_ARG, NSA_ERR_UNSUPPORTED, NSA_ERR_CUDA, NSA_ERR_TIMEOUT = range(5)
_STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA_ERROR", 4: "TIMEOUT"}

SYMBOLS = ("nsa_last_error", "nsa_version", "nsa_pool", "nsa_score", "nsa_select",
           "nsa_keep_to_index", "nsa_block_sparse_attn_fwd", "nsa_forward", "nsa_forward_timed",
           "nsa_workspace_bytes", "nsa_device_status", "nsa_forward_noalloc", "nsa_plan_bytes",
           "nsa_plan_build", "nsa_forward_plan", "nsa_schedule", "nsa_radial_blocks",
           "nsa_block_sparse_attn_fwd_masked", "nsa_block_sparse_attn_bwd", "nsa_bwd_workspace_bytes",
           "nsa_block_sparse_attn_bwd_masked", "nsa_score_tc", "nsa_selftest_timeout",
           "nsa_kernel_launches")


class NsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libnsa {_STATUS.get(status, status)}: {msg}")
        self.status = status


class nsa_spec(ctypes.Structure):
    _fields_ = [("budget", ctypes.c_float), ("block_q", ctypes.c_int32),
                ("block_kv", ctypes.c_int32), ("head_shared", ctypes.c_int32),
                ("force", ctypes.c_int32)]


@dataclass(frozen=True)
class SparseSpec:
    """Mirror of selector.py's SparseSpec (score_chunk_bytes has no
    counterpart: the fused selection never materialises scores)."""
    budget: float = 0.30
    block_q: int = 128
    block_kv: int = 64
    head_shared: bool = False
    force: bool = False

    def c(self) -> nsa_spec:
        return nsa_spec(self.budget, self.block_q, self.block_kv, int(self.head_shared), int(self.force))


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_F = ctypes.c_float
_PSPEC = ctypes.POINTER(nsa_spec)
_PI64 = ctypes.POINTER(ctypes.c_int64)

_lib.nsa_last_error.restype = ctypes.c_char_p
_lib.nsa_last_error.argtypes = []
_lib.nsa_version.restype = ctypes.c_char_p
_lib.nsa_version.argtypes = []
_lib.nsa_pool.restype = _I
_lib.nsa_pool.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P]
_lib.nsa_score.restype = _I
_lib.nsa_score.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P]
_lib.nsa_select.restype = _I
_lib.nsa_select.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _PSPEC, _P, _PI64, _P, _PI64,
                            _P, _P, _P, ctypes.POINTER(_I), _P, _SZ, _P]
_lib.nsa_keep_to_index.restype = _I
_lib.nsa_keep_to_index.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P]
_lib.nsa_block_sparse_attn_fwd.restype = _I
_lib.nsa_block_sparse_attn_fwd.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I,
                                           _F, _P, _P, _P, _SZ, _P]
_lib.nsa_block_sparse_attn_fwd_masked.restype = _I
_lib.nsa_block_sparse_attn_fwd_masked.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I,
                                                  _P, _PI64, _F, _P, _P, _P, _SZ, _P]
_lib.nsa_block_sparse_attn_bwd.restype = _I
_lib.nsa_block_sparse_attn_bwd.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I,
                                           _F, _P, _P, _P, _P, _SZ, _P]
_lib.nsa_block_sparse_attn_bwd_masked.restype = _I
_lib.nsa_block_sparse_attn_bwd_masked.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I,
                                                  _P, _PI64, _F, _P, _P, _P, _P, _SZ, _P]
_lib.nsa_score_tc.restype = _I
_lib.nsa_score_tc.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]
_lib.nsa_bwd_workspace_bytes.restype = _SZ
_lib.nsa_bwd_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _I]
_lib.nsa_forward.restype = _I
_lib.nsa_forward.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _PSPEC, _P, _PI64, _P, _PI64,
                             _F, _P, _P, _P, _P, _SZ, _P]
_lib.nsa_forward_timed.restype = _I
_lib.nsa_forward_timed.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _PSPEC, _P, _PI64, _P, _PI64,
                                   _F, _P, _P, _P, _P, _SZ, _P, _P]
_lib.nsa_forward_noalloc.restype = _I
_lib.nsa_forward_noalloc.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _PSPEC, _P, _PI64, _P, _PI64,
                                     _F, _P, _P, _P, _P]
_lib.nsa_workspace_bytes.restype = _SZ
_lib.nsa_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _PSPEC]
_lib.nsa_device_status.restype = _I
_lib.nsa_device_status.argtypes = [_I]
_lib.nsa_selftest_timeout.restype = _I
_lib.nsa_selftest_timeout.argtypes = [_I, ctypes.c_longlong, _P]
_lib.nsa_kernel_launches.restype = ctypes.c_ulonglong
_lib.nsa_kernel_launches.argtypes = []


class nsa_plan_info(ctypes.Structure):
    _fields_ = [("batches", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("covers_everything", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_D = ctypes.c_double
_lib.nsa_plan_bytes.restype = _SZ
_lib.nsa_plan_bytes.argtypes = [_I, _I, _I, _I, _PSPEC, _PI64, _PI64]
_lib.nsa_plan_build.restype = _I
_lib.nsa_plan_build.argtypes = [_I, _I, _I, _I, _PSPEC, _P, _PI64, _P, _PI64, _P, _SZ,
                                ctypes.POINTER(nsa_plan_info), _P]
_lib.nsa_forward_plan.restype = _I
_lib.nsa_forward_plan.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _PSPEC, _P,
                                  ctypes.POINTER(nsa_plan_info), _F, _P, _P, _P, _P, _SZ, _P]
_lib.nsa_schedule.restype = _I
_lib.nsa_schedule.argtypes = [_I, _D, _D, _I, ctypes.POINTER(_D)]
_lib.nsa_radial_blocks.restype = _I
_lib.nsa_radial_blocks.argtypes = [_I, _I, _I, _D, _PSPEC, _P, _P, _P, _P, _P]


def lib() -> ctypes.CDLL:
    return _lib


def nsa_last_error() -> str:
    return _lib.nsa_last_error().decode()


def nsa_version() -> str:
    return _lib.nsa_version().decode()


def _check(status: int):
    if status != NSA_OK:
        raise NsaError(status, nsa_last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _on_caller_stream(fn):
    """Runs a wrapper under its caller's `stream` (when one is given, by
    keyword or by position), so that the tensors it allocates (workspace,
    converted masks, outputs) belong to the stream its kernels run on and the
    caching allocator does not hand their memory to another stream while
    those kernels may still use it."""
    sig = inspect.signature(fn)

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        stream = sig.bind(*args, **kwargs).arguments.get("stream")
        if stream is None:
            return fn(*args, **kwargs)
        with torch.cuda.stream(stream):
            return fn(*args, **kwargs)
    return wrapper


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _mask(m, name):
    """A pin/drop tile mask: an int8/bool CUDA tensor broadcastable to
    (B, Hs, NQ, NK); returns (tensor, strides) with zero strides on broadcast
    axes, or (None, None)."""
    if m is None:
        return None, None
    if m.dtype == torch.bool:
        m = m.to(torch.int8)
    _need_cuda(m, name)
    if m.dtype != torch.int8:
        raise TypeError(f"{name} must be int8 or bool")
    if m.dim() != 4:
        raise ValueError(f"{name} must be 4-D, broadcastable to (B, Hs, NQ, NK)")
    st = [0 if m.shape[d] == 1 else m.stride(d) for d in range(4)]
    return m, (ctypes.c_int64 * 4)(*st)


def _need_cuda(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")


def block_count(length: int, block: int) -> int:
    return (length + block - 1) // block


def nsa_workspace_bytes(B, Hq, Hkv, Sq, Skv, D, spec: SparseSpec) -> int:
    c = spec.c()
    return int(_lib.nsa_workspace_bytes(B, Hq, Hkv, Sq, Skv, D, ctypes.byref(c)))


def workspace(B, Hq, Hkv, Sq, Skv, D, spec: SparseSpec, device=None) -> torch.Tensor:
    """A caller-owned workspace buffer of the size the library asks for."""
    n = nsa_workspace_bytes(B, Hq, Hkv, Sq, Skv, D, spec)
    if n == 0:
        raise ValueError("invalid sizes for a workspace")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


@_on_caller_stream
def nsa_pool(x: torch.Tensor, block: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """selector.py pool_blocks: float32 tile means of x (B,H,S,D) bf16."""
    _need(x, torch.bfloat16, "x", 4)
    B, H, S, D = x.shape
    n = block_count(S, block)
    if out is None:
        out = torch.empty(B, H, n, D, dtype=torch.float32, device=x.device)
    _need(out, torch.float32, "out", 4)
    _check(_lib.nsa_pool(_ptr(x), B, H, S, D, block, _ptr(out), _stream(stream)))
    return out


@_on_caller_stream
def nsa_score(pq: torch.Tensor, pk: torch.Tensor, head_shared: bool = False, out=None, stream=None):
    """selector.py score_blocks over pooled tensors: (B,Hs,NQ,NK) float32."""
    _need(pq, torch.float32, "pq", 4)
    _need(pk, torch.float32, "pk", 4)
    B, Hq, NQ, D = pq.shape
    Hkv, NK = pk.shape[1], pk.shape[2]
    Hs = 1 if head_shared else Hq
    if out is None:
        out = torch.empty(B, Hs, NQ, NK, dtype=torch.float32, device=pq.device)
    _check(_lib.nsa_score(_ptr(pq), _ptr(pk), B, Hq, Hkv, NQ, NK, D, int(head_shared), _ptr(out),
                          _stream(stream)))
    return out


@_on_caller_stream
def nsa_score_tc(pq: torch.Tensor, pk: torch.Tensor, stream=None) -> torch.Tensor:
    """Per-head pooled scores from the tensor-core (3xTF32) kernel: f32
    (B, Hq, NQ, NK) (a view of the (B, Hq, NQ, NK rounded up to 128) output)."""
    _need(pq, torch.float32, "pq", 4)
    _need(pk, torch.float32, "pk", 4)
    B, Hq, NQ, D = pq.shape
    Hkv, NK = pk.shape[1], pk.shape[2]
    nkp = (NK + 127) // 128 * 128
    out = torch.zeros(B, Hq, NQ, nkp, dtype=torch.float32, device=pq.device)
    half = (B * Hkv * NK * D * 4 + 255) // 256 * 256
    ws = torch.empty(2 * half, dtype=torch.uint8, device=pq.device)
    _check(_lib.nsa_score_tc(_ptr(pq), _ptr(pk), B, Hq, Hkv, NQ, NK, D, _ptr(out), _ptr(ws), ws.numel(),
                             _stream(stream)))
    return out[..., :NK]


@_on_caller_stream
def nsa_select(pq: torch.Tensor, pk: torch.Tensor, spec: SparseSpec, pins=None, drops=None,
               ws: torch.Tensor | None = None, stream=None):
    """selector.py selection_plan + select_blocks, fused with scoring.

    Returns (keep int8 (B,Hs,NQ,NK), kv_count int32 (B,Hs,NQ), kv_index
    uint16-as-int16 (B,Hs,NQ,NK), is_dense bool). is_dense mirrors the page's
    `None`: when True (only possible with force off) the caller attends densely.
    """
    _need(pq, torch.float32, "pq", 4)
    _need(pk, torch.float32, "pk", 4)
    B, Hq, NQ, D = pq.shape
    Hkv, NK = pk.shape[1], pk.shape[2]
    Hs = 1 if spec.head_shared else Hq
    dev = pq.device
    keep = torch.empty(B, Hs, NQ, NK, dtype=torch.int8, device=dev)
    count = torch.empty(B, Hs, NQ, dtype=torch.int32, device=dev)
    index = torch.empty(B, Hs, NQ, NK, dtype=torch.int16, device=dev)
    if ws is None:
        # the library's size for these tile counts (covers nsa_select's layout)
        ws = workspace(B, Hq, Hkv, NQ * spec.block_q, NK * spec.block_kv, D, spec, dev)
    pm, ps = _mask(pins, "pins")
    dm, ds = _mask(drops, "drops")
    dense = ctypes.c_int(0)
    c = spec.c()
    _check(_lib.nsa_select(_ptr(pq), _ptr(pk), B, Hq, Hkv, NQ, NK, D, ctypes.byref(c),
                           _ptr(pm), ps, _ptr(dm), ds, _ptr(keep), _ptr(count), _ptr(index),
                           ctypes.byref(dense), _ptr(ws), ws.numel(), _stream(stream)))
    return keep, count, index, bool(dense.value)


@_on_caller_stream
def nsa_keep_to_index(keep: torch.Tensor, stream=None):
    _need(keep, torch.int8, "keep", 4)
    B, Hs, NQ, NK = keep.shape
    count = torch.empty(B, Hs, NQ, dtype=torch.int32, device=keep.device)
    index = torch.empty(B, Hs, NQ, NK, dtype=torch.int16, device=keep.device)
    _check(_lib.nsa_keep_to_index(_ptr(keep), B, Hs, NQ, NK, _ptr(count), _ptr(index), _stream(stream)))
    return count, index


@_on_caller_stream
def nsa_block_sparse_attn_fwd(q, k, v, keep, scale: float, block_q: int = 128, block_kv: int = 64,
                              out=None, lse=None, ws=None, stream=None):
    """Attention over the kept tiles of `keep` (int8 (B,Hs,NQ,NK), Hs in
    {1, Hq}; None = dense). Returns (out bf16 (B,Hq,Sq,D), lse f32 (B,Hq,Sq))."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n, 4)
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    Hs = 1
    if keep is not None:
        _need(keep, torch.int8, "keep", 4)
        Hs = keep.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(B, Hq, Hkv, Sq, Skv, D, SparseSpec(1.0, block_q, block_kv), q.device)
    _check(_lib.nsa_block_sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D,
                                          _ptr(keep), Hs, block_q, block_kv, float(scale), _ptr(out),
                                          _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def _key_mask(kmask, B, Hkv, Skv):
    """A key-token mask: int8/bool CUDA tensor broadcastable to (B, Hkv, Skv);
    returns (tensor, strides) with zero strides on broadcast axes, or
    (None, None)."""
    if kmask is None:
        return None, None
    if kmask.dtype == torch.bool:
        kmask = kmask.to(torch.int8)
    _need_cuda(kmask, "kmask")
    if kmask.dtype != torch.int8 or kmask.dim() != 3:
        raise TypeError("kmask must be an int8 or bool 3-D tensor broadcastable to (B, Hkv, Skv)")
    for d, n in enumerate((B, Hkv, Skv)):
        if kmask.shape[d] not in (1, n):
            raise ValueError(f"kmask shape {tuple(kmask.shape)} does not broadcast to {(B, Hkv, Skv)}")
    return kmask, (ctypes.c_int64 * 3)(*[0 if kmask.shape[d] == 1 else kmask.stride(d) for d in range(3)])


@_on_caller_stream
def nsa_block_sparse_attn_fwd_masked(q, k, v, keep, kmask, scale: float, block_q: int = 128,
                                     block_kv: int = 64, out=None, lse=None, ws=None, stream=None):
    """nsa_block_sparse_attn_fwd with a key-token mask: `kmask` int8/bool
    CUDA tensor broadcastable to (B, Hkv, Skv), nonzero = the key token takes
    part (None = no mask). Returns (out, lse); a row whose allowed keys are
    all masked gets out 0 and lse -inf."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n, 4)
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    Hs = 1
    if keep is not None:
        _need(keep, torch.int8, "keep", 4)
        Hs = keep.shape[1]
    kmask, kst = _key_mask(kmask, B, Hkv, Skv)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(B, Hq, Hkv, Sq, Skv, D, SparseSpec(1.0, block_q, block_kv), q.device)
    _check(_lib.nsa_block_sparse_attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D,
                                                 _ptr(keep), Hs, block_q, block_kv, _ptr(kmask), kst,
                                                 float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                                 _stream(stream)))
    return out, lse


def bwd_workspace(B, Hq, Hkv, Sq, Skv, D, Hs, device):
    n = _lib.nsa_bwd_workspace_bytes(B, Hq, Hkv, Sq, Skv, D, Hs)
    if n == 0:
        raise ValueError("invalid sizes for nsa_bwd_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


@_on_caller_stream
def nsa_block_sparse_attn_bwd(q, k, v, out, lse, dout, keep, scale: float, block_q: int = 128,
                              block_kv: int = 64, dq=None, dk=None, dv=None, ws=None, stream=None, kmask=None):
    """Gradients of nsa_block_sparse_attn_fwd (or, with `kmask`, of
    nsa_block_sparse_attn_fwd_masked) for the upstream gradient `dout` (bf16
    (B,Hq,Sq,D)); `out` and `lse` are that forward's outputs for the same q,
    k, v, keep, mask and scale. Returns (dq, dk, dv) bf16."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, torch.bfloat16, n, 4)
    _need(lse, torch.float32, "lse", 3)
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    if tuple(out.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("out and dout must have q's shape, lse (B, Hq, Sq)")
    Hs = 1
    if keep is not None:
        _need(keep, torch.int8, "keep", 4)
        Hs = keep.shape[1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        ws = bwd_workspace(B, Hq, Hkv, Sq, Skv, D, Hs, q.device)
    kmask, kst = _key_mask(kmask, B, Hkv, Skv)
    _check(_lib.nsa_block_sparse_attn_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), B, Hq,
                                                 Hkv, Sq, Skv, D, _ptr(keep), Hs, block_q, block_kv, _ptr(kmask), kst,
                                                 float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                                                 _stream(stream)))
    return dq, dk, dv


@_on_caller_stream
def nsa_forward(q, k, v, spec: SparseSpec, scale: float | None = None, pins=None, drops=None,
                keep_out: torch.Tensor | None = None, out=None, lse=None, ws=None, stream=None,
                events=None):
    """The whole path: pool, fused score + plan + top-k keep, attention over
    kept tiles. Returns (out, lse). Pass `keep_out` (int8 (B,Hs,NQ,NK)) to
    also receive the keep tensor. `events`: optional 4 torch.cuda.Event (or
    None) recorded before pooling, after pooling, after selection and after
    attention (nsa_forward_timed); a middle event serialises that kernel
    boundary, so time whole steps with the middle entries None."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n, 4)
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    if keep_out is not None:
        _need(keep_out, torch.int8, "keep_out", 4)
    if ws is None:
        ws = workspace(B, Hq, Hkv, Sq, Skv, D, spec, q.device)
    pm, ps = _mask(pins, "pins")
    dm, ds = _mask(drops, "drops")
    c = spec.c()
    if events is None:
        _check(_lib.nsa_forward(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D, ctypes.byref(c),
                                _ptr(pm), ps, _ptr(dm), ds, float(scale), _ptr(out), _ptr(lse),
                                _ptr(keep_out), _ptr(ws), ws.numel(), _stream(stream)))
    else:
        if len(events) != 4:
            raise ValueError("events: 4 torch.cuda.Event (or None) expected")
        for e in events:  # torch creates the event handle on first record
            if e is not None and e.cuda_event == 0:
                e.record(stream)
        ev = (ctypes.c_void_p * 4)(*[None if e is None else e.cuda_event for e in events])
        _check(_lib.nsa_forward_timed(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D, ctypes.byref(c),
                                      _ptr(pm), ps, _ptr(dm), ds, float(scale), _ptr(out), _ptr(lse),
                                      _ptr(keep_out), _ptr(ws), ws.numel(), ev, _stream(stream)))
    return out, lse


def nsa_device_status(clear: bool = True) -> None:
    """Raises NsaError(TIMEOUT) if a kernel's bounded wait gave up."""
    _check(_lib.nsa_device_status(int(clear)))


@_on_caller_stream
def nsa_selftest_timeout(which: int, limit_cycles: int, stream=None) -> None:
    """Enqueues the kernel whose one bounded wait runs out (which 0: an
    mbarrier, site 0x70; 1: a counter, site 0x71) after limit_cycles SM
    cycles; nsa_device_status() then raises NsaError(TIMEOUT)."""
    _check(_lib.nsa_selftest_timeout(int(which), int(limit_cycles), _stream(stream)))


def nsa_kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(_lib.nsa_kernel_launches())


NOALLOC_SCRATCH_BYTES = 16 << 20


@_on_caller_stream
def nsa_forward_noalloc(q, k, v, spec: SparseSpec, scale: float | None = None, pins=None, drops=None,
                        keep_out: torch.Tensor | None = None, out=None, lse=None, stream=None):
    """nsa_forward without a workspace: the library's fixed device scratch
    array (NOALLOC_SCRATCH_BYTES) is used instead, for callers that may not
    allocate. Calls that overlap on the GPU share that array and race."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n, 4)
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    pm, ps = _mask(pins, "pins")
    dm, ds = _mask(drops, "drops")
    c = spec.c()
    _check(_lib.nsa_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D, ctypes.byref(c),
                                    _ptr(pm), ps, _ptr(dm), ds, float(scale), _ptr(out), _ptr(lse),
                                    _ptr(keep_out), _stream(stream)))
    return out, lse


# ------------------------------------------------------------ plans


@dataclass
class Plan:
    """A built selection plan (selector.py selection_plan + plan_cache): the
    caller-owned buffer and its extents. ``state`` (Bp,Hp,NQ,NK) int8,
    ``candidates`` and ``budget_counts`` (Bp,Hp,NQ) int32 are views into it."""
    buf: torch.Tensor
    info: nsa_plan_info
    state: torch.Tensor
    candidates: torch.Tensor
    budget_counts: torch.Tensor

    @property
    def covers_everything(self) -> bool:
        return bool(self.info.covers_everything)


def _align256(n: int) -> int:
    return (n + 255) // 256 * 256


@_on_caller_stream
def nsa_plan_build(B: int, Hq: int, Sq: int, Skv: int, spec: SparseSpec, pins=None, drops=None,
                   device=None, stream=None) -> Plan:
    """Builds the plan on the device; reads covers_everything back once."""
    pm, ps = _mask(pins, "pins")
    dm, ds = _mask(drops, "drops")
    c = spec.c()
    n = int(_lib.nsa_plan_bytes(B, Hq, Sq, Skv, ctypes.byref(c), ps, ds))
    if n == 0:
        raise ValueError("invalid sizes for a plan")
    dev = device or (pm.device if pm is not None else (dm.device if dm is not None else "cuda"))
    buf = torch.empty(n, dtype=torch.uint8, device=dev)
    info = nsa_plan_info()
    _check(_lib.nsa_plan_build(B, Hq, Sq, Skv, ctypes.byref(c), _ptr(pm), ps, _ptr(dm), ds, _ptr(buf), n,
                               ctypes.byref(info), _stream(stream)))
    NQ, NK = block_count(Sq, spec.block_q), block_count(Skv, spec.block_kv)
    rows = info.batches * info.heads * NQ
    o_state = 256
    o_cnt = o_state + _align256(rows * NK)
    o_k = o_cnt + _align256(rows * 4)
    state = buf[o_state:o_state + rows * NK].view(torch.int8).view(info.batches, info.heads, NQ, NK)
    cand = buf[o_cnt:o_cnt + rows * 4].view(torch.int32).view(info.batches, info.heads, NQ)
    kcnt = buf[o_k:o_k + rows * 4].view(torch.int32).view(info.batches, info.heads, NQ)
    return Plan(buf, info, state, cand, kcnt)


@_on_caller_stream
def nsa_forward_plan(q, k, v, spec: SparseSpec, plan: Plan, scale: float | None = None,
                     keep_out: torch.Tensor | None = None, out=None, lse=None, ws=None, stream=None):
    """nsa_forward with a built plan in place of pins and drops (same
    results); dense attention without any scoring when the plan covers
    everything and force is off."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n, 4)
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    if keep_out is not None:
        _need(keep_out, torch.int8, "keep_out", 4)
    if ws is None:
        ws = workspace(B, Hq, Hkv, Sq, Skv, D, spec, q.device)
    c = spec.c()
    _check(_lib.nsa_forward_plan(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D, ctypes.byref(c),
                                 _ptr(plan.buf), ctypes.byref(plan.info), float(scale), _ptr(out), _ptr(lse),
                                 _ptr(keep_out), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def nsa_schedule(steps: int, budget: float, bump: float = 0.0, bump_steps: int = 0) -> tuple:
    """selector.py schedule: per-step budgets (at most two distinct values)."""
    arr = (ctypes.c_double * max(steps, 1))()
    _check(_lib.nsa_schedule(int(steps), float(budget), float(bump), int(bump_steps), arr))
    return tuple(arr[i] for i in range(max(steps, 0)))


@_on_caller_stream
def nsa_radial_blocks(B: int, Sq: int, Skv: int, density: float, spec: SparseSpec, device=None, stream=None):
    """selector.py radial_blocks on the device: returns (keep int8 (B,1,NQ,NK),
    kv_count int32 (B,1,NQ), kv_index uint16-as-int16 (B,1,NQ,NK), width
    float64 (1,)) for the band whose kept fraction bisection aims at density."""
    NQ, NK = block_count(Sq, spec.block_q), block_count(Skv, spec.block_kv)
    dev = device or "cuda"
    keep = torch.empty(B, 1, NQ, NK, dtype=torch.int8, device=dev)
    count = torch.empty(B, 1, NQ, dtype=torch.int32, device=dev)
    index = torch.empty(B, 1, NQ, NK, dtype=torch.int16, device=dev)
    width = torch.empty(1, dtype=torch.float64, device=dev)
    c = spec.c()
    _check(_lib.nsa_radial_blocks(B, Sq, Skv, float(density), ctypes.byref(c), _ptr(width), _ptr(keep),
                                  _ptr(count), _ptr(index), _stream(stream)))
    return keep, count, index, width
