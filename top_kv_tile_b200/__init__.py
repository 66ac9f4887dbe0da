"""top_kv_tile_b200: fixed-budget block-sparse attention on B200 (sm_100a).

Block selection as defined by automatic/modules/attention/sparse/selector.py
(pool_blocks, score_blocks, selection_plan, select_blocks) and an attention
forward pass over the kept tiles, both in CUDA kernels behind the C ABI of
include/nsa.h. The Python API lives in ``top_kv_tile_b200.binding`` and is
re-exported here; it is loaded on first attribute access so that
``python -m top_kv_tile_b200.build`` can (re)build libnsa.so first. Loading
raises if libnsa.so is missing: there is no fallback implementation.
"""
from __future__ import annotations

import importlib


# submodules that must import without libnsa.so (``from top_kv_tile_b200
# import build`` asks the package for the attribute before the submodule)
_SUBMODULES = ("build", "binding", "shard")


def __getattr__(name):
    if name.startswith("__") or name in _SUBMODULES:
        raise AttributeError(name)
    mod = importlib.import_module(".binding", __name__)
    return getattr(mod, name)
