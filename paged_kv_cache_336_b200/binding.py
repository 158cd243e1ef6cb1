"""ctypes binding over libpagedkv.so (include/pagedkv.h).

Argument marshalling only: torch tensors supply device pointers, shapes and
the current CUDA stream; every step of the path runs in the library's
kernels. Nothing here computes attention, and there is no fallback: if the
shared library is missing, the first call raises ``RuntimeError``.
"""

from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedkv.so")
_lock = threading.Lock()
_lib = None

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_NO_FREE_BLOCKS = 2
PA_ERR_CUDA = 3
PA_ERR_UNSUPPORTED = 4

PA_F32 = 0
PA_BF16 = 1

DEVERR_BLOCK_ID = 0x1
DEVERR_CONTEXT_LEN = 0x2
DEVERR_SLOT = 0x4
DEVERR_COPY_PAIR = 0x8
DEVERR_TIMEOUT = 0x10


class PagedKVError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


class InvalidArgumentError(PagedKVError, ValueError):
    pass


class NoFreeBlocksError(PagedKVError):
    pass


def _status_name(status: int) -> str:
    return {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_NO_FREE_BLOCKS", 3: "PA_ERR_CUDA",
            4: "PA_ERR_UNSUPPORTED"}.get(status, f"status {status}")


class _Stats(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int64) for name in (
        "num_blocks", "free_blocks", "used_blocks", "shared_blocks", "num_seqs",
        "logical_tokens", "logical_slots", "tail_waste_slots", "cow_copies")]


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float


class StepBuffers(ctypes.Structure):
    """Mirror of pa_step_buffers_t (include/pagedkv.h)."""
    _fields_ = [
        ("max_seqs", _I), ("num_q_heads", _I), ("num_kv_heads", _I), ("head_dim", _I),
        ("block_size", _I), ("num_blocks", _I), ("max_blocks_per_seq", _I),
        ("partition_tokens", _I), ("scale", _F), ("dtype", _I),
        ("k_pool", _P), ("v_pool", _P), ("workspace", _P), ("workspace_bytes", _SZ),
        ("d_q", _P), ("d_k_new", _P), ("d_v_new", _P), ("d_out", _P),
        ("d_slots", _P), ("d_pairs", _P), ("d_tables", _P), ("d_context_lens", _P),
        ("h_slots", _P), ("h_pairs", _P), ("h_tables", _P), ("h_context_lens", _P),
        ("upload_done", _P), ("compute_done", _P), ("copy_stream", _P),
        ("download_done", _P), ("download_stream", _P),
    ]

# name -> (restype, argtypes); mirrors include/pagedkv.h
_SIGNATURES = {
    "pa_version": (ctypes.c_char_p, []),
    "pa_last_error_string": (ctypes.c_char_p, []),
    "pa_status_string": (ctypes.c_char_p, [_I]),
    "pa_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P]),
    "pa_decode_split_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "pa_decode_split_workspace_init": (_I, [_P, _SZ, _P]),
    "pa_decode_split": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _SZ,
                             _P, _P, _P]),
    "pa_decode_split_static": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                                    _P, _P, _P]),
    "pa_decode_split_static_fill_header": (_I, [ctypes.c_uint8, _P]),
    "pa_decode_shared_prefix_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "pa_decode_shared_prefix": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                                     _I, _P, _P, _P, _P, _SZ, _P, _P, _P]),
    "pa_bm_prefix_groups": (_I, [_P, _P, _I, _I, _P, _P, _P, ctypes.POINTER(_I)]),
    "pa_bm_release_before": (_I, [_P, _I64, _I64, ctypes.POINTER(_I)]),
    "pa_prefill_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "pa_prefill": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P,
                        _SZ, _P, _P, _P]),
    "pa_prefill_plan": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _I, ctypes.POINTER(_I),
                             ctypes.POINTER(_I)]),
    "pa_bm_swap_out": (_I, [_P, _I64, _P, _I, ctypes.POINTER(_I)]),
    "pa_bm_swap_in": (_I, [_P, _I64, _P, _I, ctypes.POINTER(_I)]),
    "pa_swap_out": (_I, [_P, _P, _P, _P, _P, _I, _SZ, _I, _I, _P, _P]),
    "pa_swap_in": (_I, [_P, _P, _P, _P, _P, _I, _SZ, _I, _I, _P, _P]),
    "pa_decode_split_window": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                                    _I, _P, _SZ, _P, _P, _P]),
    "pa_kv_append": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "pa_copy_blocks": (_I, [_P, _P, _P, _I, _SZ, _I, _P, _P]),
    "pa_bm_create": (_I, [_I, _I, _I, _P, ctypes.POINTER(_P)]),
    "pa_bm_destroy": (_I, [_P]),
    "pa_bm_allocate": (_I, [_P, _I64, _I64]),
    "pa_bm_fork": (_I, [_P, _I64, _I64]),
    "pa_bm_append_slot": (_I, [_P, _I64, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                               ctypes.POINTER(_I64)]),
    "pa_bm_append_slots": (_I, [_P, _P, _I, _P, _P, ctypes.POINTER(_I)]),
    "pa_bm_can_append": (_I, [_P, _P, _I, ctypes.POINTER(_I)]),
    "pa_bm_free": (_I, [_P, _I64]),
    "pa_bm_block_table": (_I, [_P, _I64, _P, _I, ctypes.POINTER(_I)]),
    "pa_bm_context_len": (_I, [_P, _I64, ctypes.POINTER(_I64)]),
    "pa_bm_export": (_I, [_P, _P, _I, _P, _P, ctypes.c_int32]),
    "pa_bm_refcount": (_I, [_P, _I, ctypes.POINTER(_I)]),
    "pa_bm_free_queue": (_I, [_P, _P, _I, ctypes.POINTER(_I)]),
    "pa_bm_stats": (_I, [_P, ctypes.POINTER(_Stats)]),
    "pa_decode_step_h2d_bytes": (_SZ, [ctypes.POINTER(StepBuffers), _I, _I]),
    "pa_decode_step_d2h_bytes": (_SZ, [ctypes.POINTER(StepBuffers), _I]),
    "pa_decode_step": (_I, [_P, ctypes.POINTER(StepBuffers), _P, _I, _P, _P, _P, _P,
                            ctypes.POINTER(_I), _I, _P, _P]),
    "pa_step_pipeline_create": (_I, [ctypes.POINTER(StepBuffers), _P, _P]),
    "pa_step_pipeline_destroy": (_I, [ctypes.POINTER(StepBuffers)]),
}


def library():
    """Load libpagedkv.so once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with `python -m paged_kv_cache_336_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _check(status: int) -> None:
    if status == PA_OK:
        return
    msg = library().pa_last_error_string().decode(errors="replace")
    if status == PA_ERR_NO_FREE_BLOCKS:
        raise NoFreeBlocksError(status, msg)
    if status == PA_ERR_INVALID_ARG:
        raise InvalidArgumentError(status, msg)
    raise PagedKVError(status, msg)


# ---------------------------------------------------------------------------
# Kernel calls. Tensors are torch tensors on the current CUDA device.

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise InvalidArgumentError(PA_ERR_INVALID_ARG, f"unsupported dtype {t.dtype}")


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream_ptr(stream) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _require_cuda(*tensors):
    for t in tensors:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise InvalidArgumentError(PA_ERR_INVALID_ARG, "tensors must be contiguous CUDA tensors")


def _decode_common(q, k_pool, v_pool, block_tables, context_lens, out):
    torch = _torch()
    _require_cuda(q, k_pool, v_pool, block_tables, context_lens, out)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "block_tables and context_lens must be int32")
    if not (q.dtype == k_pool.dtype == v_pool.dtype == out.dtype):
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "q, pools and out must share one dtype")
    if q.dim() != 3 or k_pool.dim() != 4 or k_pool.shape != v_pool.shape or out.shape != q.shape:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "bad tensor ranks/shapes")
    B, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_pool.shape
    if D2 != D or block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "shape mismatch")
    return B, Hq, D, NB, Hkv, BS, block_tables.shape[1]


def decode(q, k_pool, v_pool, block_tables, context_lens, scale: float, out=None,
           dev_err=None, stream=None):
    """pa_decode: out[s, h] = softmax(scale * K_s q[s, h]) V_s over the paged cache."""
    torch = _torch()
    if out is None:
        out = torch.empty_like(q)
    B, Hq, D, NB, Hkv, BS, MBS = _decode_common(q, k_pool, v_pool, block_tables, context_lens, out)
    _check(library().pa_decode(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv,
        D, BS, NB, MBS, float(scale), _dtype_code(q), _ptr(out), _ptr(dev_err),
        _stream_ptr(stream)))
    return out


def decode_split_workspace_size(num_seqs, num_q_heads, head_dim, block_size,
                                max_blocks_per_seq, partition_tokens) -> int:
    n = library().pa_decode_split_workspace_size(num_seqs, num_q_heads, head_dim, block_size,
                                                 max_blocks_per_seq, partition_tokens)
    if n == 0:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "bad workspace size arguments")
    return int(n)


class SplitWorkspace:
    """Device workspace for pa_decode_split (zero header), owned by torch."""

    def __init__(self, num_seqs, num_q_heads, head_dim, block_size, max_blocks_per_seq,
                 partition_tokens, device=None, stream=None):
        torch = _torch()
        self.nbytes = decode_split_workspace_size(num_seqs, num_q_heads, head_dim, block_size,
                                                  max_blocks_per_seq, partition_tokens)
        self.buffer = torch.empty(self.nbytes + 256, dtype=torch.uint8,
                                  device=device or torch.device("cuda"))
        base = self.buffer.data_ptr()
        self.ptr = (base + 255) & ~255
        _check(library().pa_decode_split_workspace_init(self.ptr, self.nbytes, _stream_ptr(stream)))
        self.partition_tokens = partition_tokens


def decode_split(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                 partition_tokens: int = 512, out=None, workspace: SplitWorkspace | None = None,
                 dev_err=None, stream=None):
    """pa_decode_split: the same result via context partitions and an LSE merge."""
    torch = _torch()
    if out is None:
        out = torch.empty_like(q)
    B, Hq, D, NB, Hkv, BS, MBS = _decode_common(q, k_pool, v_pool, block_tables, context_lens, out)
    if workspace is None:
        workspace = SplitWorkspace(B, Hq, D, BS, MBS, partition_tokens, q.device, stream)
    _check(library().pa_decode_split(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv,
        D, BS, NB, MBS, float(scale), _dtype_code(q), int(partition_tokens), workspace.ptr,
        workspace.nbytes, _ptr(out), _ptr(dev_err), _stream_ptr(stream)))
    return out


def decode_split_window(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                        window: int, partition_tokens: int = 512, out=None,
                        workspace: SplitWorkspace | None = None, dev_err=None, stream=None):
    """pa_decode_split_window: attention over the last ``window`` tokens only."""
    torch = _torch()
    if out is None:
        out = torch.empty_like(q)
    B, Hq, D, NB, Hkv, BS, MBS = _decode_common(q, k_pool, v_pool, block_tables, context_lens, out)
    if workspace is None:
        workspace = SplitWorkspace(B, Hq, D, BS, MBS, partition_tokens, q.device, stream)
    _check(library().pa_decode_split_window(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv,
        D, BS, NB, MBS, float(scale), _dtype_code(q), int(partition_tokens), int(window),
        workspace.ptr, workspace.nbytes, _ptr(out), _ptr(dev_err), _stream_ptr(stream)))
    return out


def _swap(fn_name, src_k, src_v, dst_k, dst_v, pairs, pool, host, dev_err, stream):
    torch = _torch()
    if pairs.dtype != torch.int64 or pairs.dim() != 2 or pairs.shape[1] != 2 or not pairs.is_cuda:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "pairs must be a CUDA int64 [n, 2] tensor")
    if host.is_cuda or not host.is_pinned():
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "host buffers must be pinned CPU tensors")
    if host.shape[1:] != pool.shape[1:] or host.dtype != pool.dtype:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "host buffer must be [slots, *block shape]")
    block_bytes = pool[0].numel() * pool.element_size()
    _check(getattr(library(), fn_name)(
        _ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v), _ptr(pairs), pairs.shape[0],
        block_bytes, pool.shape[0], host.shape[0], _ptr(dev_err), _stream_ptr(stream)))


def swap_out(k_pool, v_pool, host_k, host_v, pairs, dev_err=None, stream=None):
    """pa_swap_out: pairs (device block, host slot) copy whole blocks to pinned host buffers."""
    _swap("pa_swap_out", k_pool, v_pool, host_k, host_v, pairs, k_pool, host_k, dev_err, stream)


def swap_in(host_k, host_v, k_pool, v_pool, pairs, dev_err=None, stream=None):
    """pa_swap_in: pairs (host slot, device block) copy whole blocks back to the pools."""
    _swap("pa_swap_in", host_k, host_v, k_pool, v_pool, pairs, k_pool, host_k, dev_err, stream)


def prefill_workspace(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim, block_size,
                      max_blocks_per_seq, partition_tokens, device=None) -> "Workspace":
    n = library().pa_prefill_workspace_size(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim,
                                            block_size, max_blocks_per_seq, partition_tokens)
    if n == 0:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "bad workspace size arguments")
    return Workspace(n, device)


def prefill(q, k_pool, v_pool, block_tables, context_lens, query_lens, scale: float,
            partition_tokens: int = 2048, out=None, workspace=None, dev_err=None, stream=None):
    """pa_prefill: causal attention of each sequence's last query_lens[s]
    tokens over its paged context. context_lens / query_lens: host int32
    arrays; q, out: [sum(query_lens), num_q_heads, head_dim]."""
    import numpy as np
    torch = _torch()
    _require_cuda(q, k_pool, v_pool, block_tables)
    if out is None:
        out = torch.empty_like(q)
    ctx = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    qlen = np.ascontiguousarray(np.asarray(query_lens, dtype=np.int32))
    total, Hq, D = q.shape
    NB, Hkv, BS, _ = k_pool.shape
    B, MBS = block_tables.shape
    if block_tables.dtype != torch.int32 or ctx.shape != (B,) or qlen.shape != (B,):
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "bad tables or length arrays")
    if workspace is None:
        workspace = prefill_workspace(B, total, Hq, Hkv, D, BS, MBS, partition_tokens, q.device)
    _check(library().pa_prefill(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), ctx.ctypes.data, qlen.ctypes.data,
        B, total, Hq, Hkv, D, BS, NB, MBS, float(scale), _dtype_code(q), int(partition_tokens),
        workspace.ptr, workspace.nbytes, _ptr(out), _ptr(dev_err), _stream_ptr(stream)))
    return out


def prefill_plan(context_lens, query_lens, num_q_heads: int, num_kv_heads: int, block_size: int,
                 partition_tokens: int, max_ctas: int = 0):
    """pa_prefill_plan (host only): the tcgen05 prefill kernel's items as an
    int32 array [n, 6] of (seq, first query token, query tokens, kv head,
    partition, cta), in the order the kernel runs them, and the grid size."""
    import numpy as np
    ctx = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    qlen = np.ascontiguousarray(np.asarray(query_lens, dtype=np.int32))
    if ctx.shape != qlen.shape or ctx.ndim != 1:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "bad length arrays")
    n, grid = ctypes.c_int(0), ctypes.c_int(0)
    args = (ctx.ctypes.data, qlen.ctypes.data, len(ctx), int(num_q_heads), int(num_kv_heads),
            int(block_size), int(partition_tokens), int(max_ctas))
    _check(library().pa_prefill_plan(*args, None, 0, ctypes.byref(n), ctypes.byref(grid)))
    items = np.zeros((n.value, 6), dtype=np.int32)
    _check(library().pa_prefill_plan(*args, items.ctypes.data, n.value, ctypes.byref(n),
                                     ctypes.byref(grid)))
    return items, grid.value


class Workspace:
    """Caller-owned, 256-byte aligned device workspace, zeroed once (the
    contract of pa_decode_split_workspace_init)."""

    def __init__(self, nbytes: int, device=None, stream=None):
        torch = _torch()
        self.nbytes = int(nbytes)
        self.buffer = torch.empty(self.nbytes + 256, dtype=torch.uint8,
                                  device=device or torch.device("cuda"))
        self.ptr = (self.buffer.data_ptr() + 255) & ~255
        _check(library().pa_decode_split_workspace_init(self.ptr, self.nbytes, _stream_ptr(stream)))


def shared_prefix_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                            max_blocks_per_seq, partition_tokens, device=None) -> Workspace:
    n = library().pa_decode_shared_prefix_workspace_size(
        num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
        partition_tokens)
    if n == 0:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "bad workspace size arguments")
    return Workspace(n, device)


def decode_shared_prefix(q, k_pool, v_pool, block_tables, context_lens, scale: float, groups,
                         partition_tokens: int = 512, out=None, workspace: Workspace | None = None,
                         dev_err=None, stream=None):
    """pa_decode_shared_prefix. ``groups`` = (offsets, members, blocks) as host
    int32 arrays, e.g. from BlockManager.prefix_groups()."""
    import numpy as np
    torch = _torch()
    if out is None:
        out = torch.empty_like(q)
    B, Hq, D, NB, Hkv, BS, MBS = _decode_common(q, k_pool, v_pool, block_tables, context_lens, out)
    offs, members, blocks = (np.ascontiguousarray(np.asarray(x, dtype=np.int32)) for x in groups)
    if workspace is None:
        workspace = shared_prefix_workspace(B, Hq, Hkv, D, BS, MBS, partition_tokens, q.device)
    _check(library().pa_decode_shared_prefix(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv,
        D, BS, NB, MBS, float(scale), _dtype_code(q), int(partition_tokens), int(blocks.shape[0]),
        offs.ctypes.data, members.ctypes.data if members.size else None,
        blocks.ctypes.data if blocks.size else None, workspace.ptr, workspace.nbytes, _ptr(out),
        _ptr(dev_err), _stream_ptr(stream)))
    return out


def kv_append(k_new, v_new, slot_mapping, k_pool, v_pool, dev_err=None, stream=None):
    """pa_kv_append: pool[slot // bs, :, slot % bs, :] = new[t] for K and V."""
    torch = _torch()
    _require_cuda(k_new, v_new, slot_mapping, k_pool, v_pool)
    if slot_mapping.dtype != torch.int64:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "slot_mapping must be int64")
    T, Hkv, D = k_new.shape
    NB, Hkv2, BS, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or v_new.shape != k_new.shape or slot_mapping.shape != (T,):
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "shape mismatch")
    _check(library().pa_kv_append(
        _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, Hkv, D, BS, NB, _dtype_code(k_new),
        _ptr(k_pool), _ptr(v_pool), _ptr(dev_err), _stream_ptr(stream)))


def copy_blocks(k_pool, v_pool, src_dst_pairs, dev_err=None, stream=None):
    """pa_copy_blocks: whole-block copies src -> dst in both pools."""
    torch = _torch()
    _require_cuda(k_pool, v_pool, src_dst_pairs)
    if src_dst_pairs.dtype != torch.int64 or src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise InvalidArgumentError(PA_ERR_INVALID_ARG, "src_dst_pairs must be int64 [n, 2]")
    NB = k_pool.shape[0]
    block_bytes = k_pool[0].numel() * k_pool.element_size()
    _check(library().pa_copy_blocks(
        _ptr(k_pool), _ptr(v_pool), _ptr(src_dst_pairs), src_dst_pairs.shape[0], block_bytes, NB,
        _ptr(dev_err), _stream_ptr(stream)))


# ---------------------------------------------------------------------------
# Host block manager.

@dataclass
class AppendResult:
    slot: int
    cow_src: int = -1
    cow_dst: int = -1


class BlockManager:
    """Handle over the C++ block manager (pa_bm_*). Not thread-safe."""

    def __init__(self, num_blocks: int, block_size: int, max_blocks_per_seq: int,
                 initial_free_order=None):
        import numpy as np
        lib = library()
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        self.max_blocks_per_seq = int(max_blocks_per_seq)
        handle = _P()
        order_ptr = None
        if initial_free_order is not None:
            self._order = np.ascontiguousarray(np.asarray(initial_free_order, dtype=np.int32))
            if self._order.shape != (self.num_blocks,):
                raise InvalidArgumentError(PA_ERR_INVALID_ARG, "initial_free_order has the wrong length")
            order_ptr = self._order.ctypes.data
        _check(lib.pa_bm_create(self.num_blocks, self.block_size, self.max_blocks_per_seq,
                                order_ptr, ctypes.byref(handle)))
        self._h = handle

    def close(self):
        if getattr(self, "_h", None):
            library().pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate(self, seq: int, num_tokens: int) -> None:
        _check(library().pa_bm_allocate(self._h, int(seq), int(num_tokens)))

    def fork(self, parent: int, child: int) -> None:
        _check(library().pa_bm_fork(self._h, int(parent), int(child)))

    def append_slot(self, seq: int) -> AppendResult:
        slot, cs, cd = _I64(), _I64(), _I64()
        _check(library().pa_bm_append_slot(self._h, int(seq), ctypes.byref(slot), ctypes.byref(cs),
                                           ctypes.byref(cd)))
        return AppendResult(slot.value, cs.value, cd.value)

    def append_slots_arrays(self, seqs):
        """Batched step; returns (slots int64 [n], cow_pairs int64 [k, 2]) as numpy."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(seqs, dtype=np.int64))
        n = ids.shape[0]
        slots = np.empty(n, dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        k = _I()
        _check(library().pa_bm_append_slots(self._h, ids.ctypes.data, n, slots.ctypes.data,
                                            pairs.ctypes.data, ctypes.byref(k)))
        return slots, pairs[:k.value].copy()

    def append_slots(self, seqs) -> list[AppendResult]:
        """Batched step with per-sequence results (copy pairs matched by order)."""
        slots, pairs = self.append_slots_arrays(seqs)
        out, k = [], 0
        for s in slots:
            r = AppendResult(int(s))
            if k < len(pairs) and int(pairs[k][1]) * self.block_size == int(s) // self.block_size * self.block_size:
                r.cow_src, r.cow_dst = int(pairs[k][0]), int(pairs[k][1])
                k += 1
            out.append(r)
        return out

    def can_append(self, seqs) -> bool:
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(seqs, dtype=np.int64))
        ok = _I()
        _check(library().pa_bm_can_append(self._h, ids.ctypes.data, ids.shape[0], ctypes.byref(ok)))
        return bool(ok.value)

    def free(self, seq: int) -> None:
        _check(library().pa_bm_free(self._h, int(seq)))

    def block_table(self, seq: int) -> list[int]:
        import numpy as np
        row = np.empty(self.max_blocks_per_seq, dtype=np.int32)
        n = _I()
        _check(library().pa_bm_block_table(self._h, int(seq), row.ctypes.data, row.shape[0],
                                           ctypes.byref(n)))
        return [int(x) for x in row[:n.value]]

    def context_len(self, seq: int) -> int:
        c = _I64()
        _check(library().pa_bm_context_len(self._h, int(seq), ctypes.byref(c)))
        return int(c.value)

    def export(self, seqs, pad_value: int = -1):
        """(tables int32 [n, max_blocks_per_seq], context_lens int32 [n]) as numpy."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(seqs, dtype=np.int64))
        n = ids.shape[0]
        tables = np.empty((n, self.max_blocks_per_seq), dtype=np.int32)
        ctx = np.empty(n, dtype=np.int32)
        _check(library().pa_bm_export(self._h, ids.ctypes.data, n, tables.ctypes.data,
                                      ctx.ctypes.data, int(pad_value)))
        return tables, ctx

    def swap_out(self, seq: int) -> list[int]:
        """pa_bm_swap_out: the sequence's table at swap-out (blocks to copy out)."""
        import numpy as np
        buf = np.empty(self.max_blocks_per_seq, dtype=np.int32)
        n = _I()
        _check(library().pa_bm_swap_out(self._h, int(seq), buf.ctypes.data, buf.shape[0],
                                        ctypes.byref(n)))
        return [int(x) for x in buf[:n.value]]

    def swap_in(self, seq: int) -> list[int]:
        """pa_bm_swap_in: the new table (blocks to copy the host copies into)."""
        import numpy as np
        buf = np.empty(self.max_blocks_per_seq, dtype=np.int32)
        n = _I()
        _check(library().pa_bm_swap_in(self._h, int(seq), buf.ctypes.data, buf.shape[0],
                                       ctypes.byref(n)))
        return [int(x) for x in buf[:n.value]]

    def release_before(self, seq: int, first_token: int) -> int:
        """pa_bm_release_before; returns the number of blocks reclaimed."""
        k = _I()
        _check(library().pa_bm_release_before(self._h, int(seq), int(first_token), ctypes.byref(k)))
        return int(k.value)

    def prefix_groups(self, seqs, min_shared_blocks: int = 1):
        """pa_bm_prefix_groups: (offsets [g+1], members [m], blocks [g]) int32
        numpy arrays; members are positions in ``seqs``."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(seqs, dtype=np.int64))
        n = ids.shape[0]
        offs = np.zeros(n + 1, dtype=np.int32)
        members = np.zeros(max(n, 1), dtype=np.int32)
        blocks = np.zeros(max(n, 1), dtype=np.int32)
        k = _I()
        _check(library().pa_bm_prefix_groups(self._h, ids.ctypes.data, n, int(min_shared_blocks),
                                             offs.ctypes.data, members.ctypes.data,
                                             blocks.ctypes.data, ctypes.byref(k)))
        g = k.value
        return offs[:g + 1].copy(), members[:offs[g]].copy(), blocks[:g].copy()

    def refcount_of(self, block: int) -> int:
        rc = _I()
        _check(library().pa_bm_refcount(self._h, int(block), ctypes.byref(rc)))
        return int(rc.value)

    def free_queue_list(self) -> list[int]:
        import numpy as np
        buf = np.empty(self.num_blocks, dtype=np.int32)
        n = _I()
        _check(library().pa_bm_free_queue(self._h, buf.ctypes.data, buf.shape[0], ctypes.byref(n)))
        return [int(x) for x in buf[:n.value]]

    def num_free(self) -> int:
        return self.stats()["free_blocks"]

    def stats(self) -> dict:
        st = _Stats()
        _check(library().pa_bm_stats(self._h, ctypes.byref(st)))
        return {name: int(getattr(st, name)) for name, _ in _Stats._fields_}


# ---------------------------------------------------------------------------
# One whole decode step from host buffers (pa_decode_step).

class DecodeStepper:
    """Owns the staging buffers of pa_decode_step for one cache and manager.

    Device staging is torch-allocated once; host staging is page-locked. Each
    ``step`` call is one C call: manager step, uploads, copies, append, split
    decode, download (and, by default, stream synchronisation)."""

    def __init__(self, bm: "BlockManager", k_pool, v_pool, num_q_heads: int, scale: float,
                 max_seqs: int, partition_tokens: int = 512, copy_stream=None,
                 download_stream=None):
        """copy_stream: a torch.cuda.Stream for the uploads (pipelined steps,
        see pa_step_pipeline_create), download_stream one for the download
        (made here when not given); None runs everything on the step's stream."""
        torch = _torch()
        _require_cuda(k_pool, v_pool)
        NB, Hkv, BS, D = k_pool.shape
        dev = k_pool.device
        self.bm = bm
        self.k_pool, self.v_pool = k_pool, v_pool
        self.dtype = k_pool.dtype
        mbs = bm.max_blocks_per_seq
        self.ws = SplitWorkspace(max_seqs, num_q_heads, D, BS, mbs, partition_tokens, dev)
        self.d_q = torch.empty(max_seqs, num_q_heads, D, dtype=self.dtype, device=dev)
        self.d_out = torch.empty_like(self.d_q)
        self.d_k_new = torch.empty(max_seqs, Hkv, D, dtype=self.dtype, device=dev)
        self.d_v_new = torch.empty_like(self.d_k_new)
        # the four small staging arrays back to back (slots | pairs | lengths |
        # tables) on both sides, so one upload carries them
        nbytes = max_seqs * (8 + 16 + 4) + max_seqs * mbs * 4
        self.d_pack = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.h_pack = torch.empty(nbytes, dtype=torch.uint8).pin_memory()

        def views(buf):
            o1, o2, o3 = max_seqs * 8, max_seqs * 24, max_seqs * 28
            return (buf[:o1].view(torch.int64), buf[o1:o2].view(torch.int64).view(max_seqs, 2),
                    buf[o2:o3].view(torch.int32), buf[o3:].view(torch.int32).view(max_seqs, mbs))

        self.d_slots, self.d_pairs, self.d_ctx, self.d_tables = views(self.d_pack)
        self.h_slots, self.h_pairs, self.h_ctx, self.h_tables = views(self.h_pack)
        b = StepBuffers()
        b.max_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim = max_seqs, num_q_heads, Hkv, D
        b.block_size, b.num_blocks, b.max_blocks_per_seq = BS, NB, mbs
        b.partition_tokens, b.scale, b.dtype = partition_tokens, float(scale), _dtype_code(k_pool)
        b.k_pool, b.v_pool = _ptr(k_pool), _ptr(v_pool)
        b.workspace, b.workspace_bytes = self.ws.ptr, self.ws.nbytes
        b.d_q, b.d_k_new, b.d_v_new, b.d_out = (_ptr(self.d_q), _ptr(self.d_k_new),
                                                _ptr(self.d_v_new), _ptr(self.d_out))
        b.d_slots, b.d_pairs = _ptr(self.d_slots), _ptr(self.d_pairs)
        b.d_tables, b.d_context_lens = _ptr(self.d_tables), _ptr(self.d_ctx)
        b.h_slots, b.h_pairs = _ptr(self.h_slots), _ptr(self.h_pairs)
        b.h_tables, b.h_context_lens = _ptr(self.h_tables), _ptr(self.h_ctx)
        self.buffers = b
        self.copy_stream = copy_stream
        if copy_stream is not None:
            self.download_stream = download_stream or torch.cuda.Stream(device=dev)
            _check(library().pa_step_pipeline_create(ctypes.byref(self.buffers),
                                                     _stream_ptr(copy_stream),
                                                     _stream_ptr(self.download_stream)))

    def __del__(self):
        try:
            if getattr(self, "copy_stream", None) is not None:
                library().pa_step_pipeline_destroy(ctypes.byref(self.buffers))
        except Exception:
            pass

    def h2d_bytes(self, n: int, num_copies: int) -> int:
        return int(library().pa_decode_step_h2d_bytes(ctypes.byref(self.buffers), n, num_copies))

    def d2h_bytes(self, n: int) -> int:
        return int(library().pa_decode_step_d2h_bytes(ctypes.byref(self.buffers), n))

    def step(self, seq_ids, q_host, k_new_host, v_new_host, out_host, synchronize: bool = True,
             dev_err=None, stream=None) -> int:
        """Runs one step; returns the number of copy-on-write copies it made.
        ``seq_ids`` is a contiguous int64 numpy array; the host tensors are CPU
        tensors (pinned for asynchronous copies) of the shapes in pagedkv.h."""
        n = int(seq_ids.shape[0])
        ncow = _I()
        _check(library().pa_decode_step(
            self.bm._h, ctypes.byref(self.buffers), seq_ids.ctypes.data, n, _ptr(q_host),
            _ptr(k_new_host), _ptr(v_new_host), _ptr(out_host), ctypes.byref(ncow),
            1 if synchronize else 0, _ptr(dev_err), _stream_ptr(stream)))
        return int(ncow.value)

