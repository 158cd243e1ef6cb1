"""GPU parity at the full sizes of the measured workloads, in the launch
configuration the bench times (block-manager step, copy-on-write copies,
append, split decode with 512-token partitions).

Every (sequence, query head) output is compared with the float64 oracle,
which walks the real block tables itself (one KV head's slice of the pools at
a time, since the pools do not fit on the host in float64); the tolerances
apply to the whole output. The copies and appends of the step are checked
bit-exactly over the whole pool: the oracle applies the same copy pairs and
slots to a snapshot taken before the step.
"""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import (as_bits, check_close, device_tables, host_slice, oracle_decode_by_kv_head,
                      setup, to_f64)

pytestmark = pytest.mark.gpu


def _check_step_bit_exact(w, k_before, v_before, k_pool, v_pool, pairs, slots, k_new, v_new):
    """Whole pools after the step == oracle.copy_blocks + oracle.kv_append
    applied to the snapshot, one KV head at a time, on raw bit patterns."""
    kn, vn = as_bits(k_new), as_bits(v_new)
    for kvh in range(w.num_kv_heads):
        kb, vb = host_slice(k_before, kvh, bits=True), host_slice(v_before, kvh, bits=True)
        oracle.copy_blocks(kb, vb, pairs)
        oracle.kv_append(kb, vb, kn[:, kvh:kvh + 1], vn[:, kvh:kvh + 1], slots)
        assert np.array_equal(kb, host_slice(k_pool, kvh, bits=True)), f"K pool, KV head {kvh}"
        assert np.array_equal(vb, host_slice(v_pool, kvh, bits=True)), f"V pool, KV head {kvh}"


def _step_and_decode(w, partition_tokens=512):
    bm, k_pool, v_pool = setup(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pairs = np.zeros((0, 2), dtype=np.int64)
    if w.step_seqs:
        k_before, v_before = k_pool.clone(), v_pool.clone()
        slots, pairs = bm.append_slots_arrays(w.step_seqs)
        k_new, v_new = workloads.draw_new_kv(w, len(w.step_seqs), device="cuda")
        if len(pairs):
            binding.copy_blocks(k_pool, v_pool, torch.from_numpy(pairs).cuda(), dev_err=err)
        binding.kv_append(k_new, v_new, torch.from_numpy(slots).cuda(), k_pool, v_pool, dev_err=err)
        torch.cuda.synchronize()
        _check_step_bit_exact(w, k_before, v_before, k_pool, v_pool, pairs, slots, k_new, v_new)
        del k_before, v_before
        torch.cuda.empty_cache()
    seqs = w.decode_seqs
    bt, ctx, tables, ctx_np = device_tables(bm, seqs)
    q = workloads.draw_queries(w, len(seqs), device="cuda")
    out = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale,
                               partition_tokens=partition_tokens, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle_decode_by_kv_head(q, k_pool, v_pool, tables, ctx_np, w.scale)
    return to_f64(out), want, len(pairs)


def test_mha_batch64():
    w = workloads.mha()
    got, want, n_cow = _step_and_decode(w)
    check_close(got, want, w.dtype, "mha")
    assert n_cow == 0


def test_gqa_batch256():
    w = workloads.gqa()
    got, want, _ = _step_and_decode(w)
    check_close(got, want, w.dtype, "gqa")


def test_prefix_sharing():
    w = workloads.prefix()
    got, want, n_cow = _step_and_decode(w)
    check_close(got, want, w.dtype, "prefix")


def test_prefix_sharing_cow_step():
    w = workloads.prefix_cow()
    got, want, n_cow = _step_and_decode(w)
    check_close(got, want, w.dtype, "prefix_cow")
    assert n_cow == 120


@pytest.mark.parametrize("bs", [16, 32])
def test_long_context_split(bs):
    w = workloads.long(block_size=bs, slack=0.1)
    got, want, _ = _step_and_decode(w)
    check_close(got, want, w.dtype, f"long bs{bs}")
