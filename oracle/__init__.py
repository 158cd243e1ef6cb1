"""CPU oracle for the paged decode-attention path: TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct statement of what the
GPU path computes. It exists so that tests, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` leg of ``bench.py`` have something independent to compare
against. Nothing in the product path (the ``paged_kv_cache_336_b200`` package,
its CUDA kernels or its C ABI) imports, calls or links it, and it imports
nothing from the product path.

Modules
-------
``paged_attention``
    Decode attention over a block-paged KV cache, written as its definition:
    gather each sequence's keys and values through its block table, then
    softmax(scale * K q) V in float64, two-pass (max, then exp/sum).
    Also the causal prefill over the paged cache (many new tokens per
    sequence), the sliding-window form (the last ``window`` tokens only), the
    partitioned form (per-partition max/sum/accumulator and a log-sum-exp
    merge), the KV-append scatter and the block copy, as plain array
    assignments.
``block_manager``
    Reference host block manager: FIFO free queue, reference counts,
    per-sequence block tables, copy-on-write on append, all-or-nothing
    failure.

Sources (web pages on PagedAttention; cited by page title and section):

* "What is PagedAttention?" (qubittool.com glossary), section "How It Works"
  (Map Logical to Physical Blocks; Share Without Mutating State).
* "PagedAttention" (kongchang.com knowledge page), "Core Facts".
* "PagedAttention: Optimizing KV Cache in vLLM" (grasp.study lesson),
  sections 2, 3 and 4.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
something other than itself (a library routine, closed forms, invariants and
a hand-worked trace under ``tests/golden/``). No function here is unpinned.
"""

from .paged_attention import (  # noqa: F401
    attention_definition,
    gather_sequence,
    paged_decode,
    paged_decode_one,
    paged_decode_window,
    paged_prefill,
    partitioned_decode_one,
    kv_append,
    copy_blocks,
)
from .block_manager import (  # noqa: F401
    BlockManager,
    InvalidArgument,
    NoFreeBlocks,
)
