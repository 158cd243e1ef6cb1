"""B200-native paged decode attention (PagedAttention's data-parallel hot path).

The compute lives in ``libpagedkv.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/pagedkv.h``); this package is a thin ctypes
binding over it plus the seeded input generators in ``workloads``. Torch is
used only to own device memory and streams.

Importing the package does not load the shared library; the first call that
needs it does, and raises ``RuntimeError`` if it has not been built
(``python -m paged_kv_cache_336_b200.build``). There is no CPU fallback.
"""

from .binding import (  # noqa: F401
    BlockManager,
    DecodeStepper,
    PagedKVError,
    NoFreeBlocksError,
    InvalidArgumentError,
    decode,
    decode_split,
    decode_split_window,
    decode_shared_prefix,
    prefill,
    decode_split_workspace_size,
    kv_append,
    copy_blocks,
    swap_out,
    swap_in,
    library,
)
