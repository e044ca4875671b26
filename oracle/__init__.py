"""CPU oracle for chunk attention over a segmented KV cache.

TEST INFRASTRUCTURE ONLY: a plain fp64 NumPy statement of what the CUDA path
computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it.  It shares no code with the library.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force, closed forms, invariants and hand-worked cases in
``tests/golden/``); none is unpinned.
"""
from .attention import (  # noqa: F401
    attend,
    block_scores,
    block_select,
    block_sparse_attention,
    lse_merge,
    pool_blocks,
    ragged_attention,
    segment_attention,
    segment_rows,
    select_topk,
    to64,
    topk_gap,
    visited_flops_ragged,
    visited_flops_segments,
    visited_flops_sparse,
)
from .compaction import compact_cache, head_frames, merge_frames  # noqa: F401
from .memory import persist_update  # noqa: F401
from .mla import latent_attention, visited_flops_latent  # noqa: F401
