"""fp64 CPU oracle for the paged-attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run anything in this package.
The product library (``paged_kv_cache_332_b200``) never calls it and shares no
code with it.

Contents
--------
``paged_attention``  plain NumPy fp64 restatement of what the path computes:
                     the KV-size formula, the block-count rule, the slot
                     scatter (reshape_and_cache), paged decode attention and
                     causal chunked-prefill attention, plus round-to-nearest-
                     even to fp16 / bf16.
``dense_attention.c`` an independent plain-C dense (contiguous, no paging)
                     attention used only to pin the NumPy oracle on tiny
                     inputs; compiled by ``__graft_entry__.build()``.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, the pages' worked example, invariants and brute force; no
function is "parity unpinned".
"""
from .paged_attention import (  # noqa: F401
    kv_cache_size_bytes, blocks_needed, slot_of, reshape_and_cache,
    kv_head_of, gather_kv, attend, paged_decode, chunked_prefill,
    round_rne, round_to, to_f64,
)
