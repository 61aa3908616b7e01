"""Oracle for the block-sparse KV attention path (fp64, CPU, slow on purpose).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product package.  It
shares no code with the CUDA library under ``block_sparse_kv_bsa_b200/``.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, invariants, brute force on tiny inputs or textbook
routines (see the test files); none is "parity unpinned".

``oracle.geometry`` holds the overlap prior g and the coverage score
(slab boxes, separating-axis test, grid IoU), in float32 with a fixed
operation order because they decide counts.
"""
from .gilbert import gilbert_cells, gilbert_perm  # noqa: F401
from .bsa import (  # noqa: F401
    BLK,
    attn,
    attn_block,
    attn_rows,
    block_scores,
    block_valid_for,
    blocks_to_tokens,
    dense_masked_attn,
    fuse_prior,
    kv_append,
    n_blocks_for,
    pool_blocks,
    route,
    tokens_to_blocks,
    top_k_with_own,
    velox_route,
    velox_route_row,
    vetted_overlap,
)
