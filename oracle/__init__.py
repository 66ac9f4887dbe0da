"""CPU oracle for fixed-budget block selection and block-sparse attention.

TEST INFRASTRUCTURE ONLY. This package is the slow, plain reference that the
CUDA library is checked against. Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it. The product path (``top_kv_tile_b200``) never imports or calls it, and it
imports nothing from the product path.

Everything is NumPy in float64, except the one place the method itself fixes
a lower precision: the per-row budget count ``ceil(candidates * budget)``,
which the selector evaluates in float32 (selection_plan in
automatic/modules/attention/sparse/selector.py).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, hand counts, brute force and library special cases; none
is "parity unpinned".
"""
from .selector import (  # noqa: F401
    SparseSpec, block_count, pool_blocks, diagonal_blocks, head_map,
    score_blocks, selection_plan, select_blocks, select_pooled, keep_to_lists,
    boundary_scores, radial_blocks, schedule, budget_count, select_rows,
)
from .attention import block_sparse_attention, attention_tiles, block_sparse_attention_bwd  # noqa: F401
