"""The no-allocation split decode entry point, pa_decode_split_static.

It exists for callers that cannot call cudaMalloc (their device memory is
owned by another allocator, or an allocation in the middle of a decode loop
is not acceptable); its scratch is a fixed array inside the library. These
tests call it through the C ABI and compare it with pa_decode_split, which
takes a caller workspace, and with the float64 oracle, within the tolerances
used by every decode test (fp32 max-abs 1e-5; bf16 max-abs 2e-2 and
mean-abs 2e-3), on two calls in a row, since the array keeps the previous
call's contents, and after the array's header was left dirty (as a call that
timed out could leave it). Oversized requests, and requests refused for any
other reason, must be turned away before anything is enqueued.

This file sorts last so that a run stopping at the first failure has run
every other test first; it also passes when run alone in a fresh process.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 16 * 1024 * 1024   # PA_STATIC_SCRATCH_BYTES in include/pagedkv.h


def _call_static(q, k_pool, v_pool, bt, ctx, scale, partition_tokens, out, err):
    lib = binding.library()
    B, Hq, D = q.shape
    NB, Hkv, BS, _ = k_pool.shape
    dtype = binding.PA_F32 if q.dtype == torch.float32 else binding.PA_BF16
    return lib.pa_decode_split_static(
        q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), bt.data_ptr(), ctx.data_ptr(), B, Hq,
        Hkv, D, BS, NB, bt.shape[1], float(scale), dtype, int(partition_tokens), out.data_ptr(),
        err.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("dtype,G", [(workloads.F32, 1), (workloads.BF16, 1), (workloads.BF16, 8)])
def test_static_scratch_matches_workspace_entry_point(dtype, G):
    for split_kernel in ("ticket", "stream"):
        os.environ["PAGEDKV_SPLIT_KERNEL"] = split_kernel
        try:
            _static_matches(dtype, G)
        finally:
            os.environ.pop("PAGEDKV_SPLIT_KERNEL", None)


def _static_matches(dtype, G):
    torch.cuda.set_device(0)
    w = workloads.random_small(31 + G, num_seqs=9, num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=128, block_size=16, dtype=dtype, max_ctx=400,
                               fixed_lens=[0, 1, 400])
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 9, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(9)))
    partition = 48  # several partitions per sequence, ragged last one
    need = binding.decode_split_workspace_size(9, 2 * G, 128, 16, bt.shape[1], partition)
    assert need <= STATIC_SCRATCH_BYTES
    ref = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=partition)
    ref_np = to_f64(ref)
    want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, w.scale)
    check_close(ref_np, want, dtype, "workspace entry point vs oracle")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        status = _call_static(q, k_pool, v_pool, bt, ctx, w.scale, partition, out, err)
        assert status == binding.PA_OK, binding.library().pa_last_error_string()
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"call {call}: device error word {int(err.item()):#x}"
        check_close(to_f64(out), ref_np, dtype, f"static scratch vs workspace, call {call}")
        check_close(to_f64(out), want, dtype, f"static scratch vs oracle, call {call}")
    assert torch.all(out[0] == 0)   # empty context


def test_static_scratch_refuses_oversized_requests():
    torch.cuda.set_device(0)
    # small real buffers; the declared sizes are refused before any launch
    q = torch.zeros(4, 64, 128, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(8, 8, 16, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(4, 8, dtype=torch.int32, device="cuda")
    ctx = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib = binding.library()
    big_seqs, mbs = 4096, 8192
    need = binding.decode_split_workspace_size(big_seqs, 64, 128, 16, mbs, 16)
    assert need > STATIC_SCRATCH_BYTES
    status = lib.pa_decode_split_static(
        q.data_ptr(), pool.data_ptr(), pool.data_ptr(), bt.data_ptr(), ctx.data_ptr(), big_seqs,
        64, 8, 128, 16, 8, mbs, 0.1, binding.PA_BF16, 16, out.data_ptr(), err.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert status == binding.PA_ERR_INVALID_ARG
    assert b"static" in lib.pa_last_error_string() and b"scratch" in lib.pa_last_error_string()
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and torch.all(out == 0)

    # more sequences than the split decode takes (4096), with scratch to
    # spare: refused by the sequence-count check, which comes before the
    # call touches the shared array
    n = 4097
    q1 = torch.zeros(n, 1, 128, dtype=torch.bfloat16, device="cuda")
    bt1 = torch.zeros(n, 1, dtype=torch.int32, device="cuda")
    ctx1 = torch.zeros(n, dtype=torch.int32, device="cuda")
    out1 = torch.zeros_like(q1)
    assert binding.decode_split_workspace_size(n, 1, 128, 16, 1, 16) <= STATIC_SCRATCH_BYTES
    status = lib.pa_decode_split_static(
        q1.data_ptr(), pool.data_ptr(), pool.data_ptr(), bt1.data_ptr(), ctx1.data_ptr(), n, 1, 1,
        128, 16, 8, 1, 0.1, binding.PA_BF16, 16, out1.data_ptr(), err.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert status == binding.PA_ERR_UNSUPPORTED
    assert b"4096" in lib.pa_last_error_string()
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and torch.all(out1 == 0)

    # a call after the refusals still matches the oracle
    _static_matches(workloads.BF16, 8)


@pytest.mark.parametrize("split_kernel", ["ticket", "stream"])
def test_static_call_after_a_dirty_header(monkeypatch, split_kernel):
    """A call that ended early (a device timeout) can leave the shared array's
    ticket counters non-zero. Each static call clears the header after its
    host checks, so a call that follows a dirty header is still correct: the
    test fills the header with 0x5A bytes (counters 0x5A5A5A5A, far past any
    ticket) through the library's test aid, then compares a static call with
    the oracle. Without the clear, the ticket kernel would find no tickets
    and leave the output unwritten."""
    monkeypatch.setenv("PAGEDKV_SPLIT_KERNEL", split_kernel)
    torch.cuda.set_device(0)
    lib = binding.library()
    w = workloads.random_small(77, num_seqs=9, num_q_heads=16, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=400,
                               fixed_lens=[0, 1, 400])
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 9, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(9)))
    want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, w.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        assert lib.pa_decode_split_static_fill_header(0x5A, stream) == binding.PA_OK
        out = torch.full_like(q, float("nan"))
        status = _call_static(q, k_pool, v_pool, bt, ctx, w.scale, 48, out, err)
        assert status == binding.PA_OK, lib.pa_last_error_string()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        check_close(to_f64(out), want, workloads.BF16, f"static call {call} after a dirty header")
