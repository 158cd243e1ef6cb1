"""Swap round trip on the GPU: a sequence is preempted (its blocks copied to
pinned host memory and reclaimed), the pool reuses the blocks, the sequence
comes back into new blocks. The host copies and the swapped-in blocks are
checked bit for bit against the oracle's gather through the old and new
tables; the decode before and after is checked against the oracle, and is
bit-identical across the swap (placement does not matter)."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,G", [(workloads.BF16, 4), (workloads.F32, 1)])
def test_swap_out_reuse_swap_in(dtype, G):
    w = workloads.random_small(90 + G, num_seqs=4, num_q_heads=2 * G, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=dtype, max_ctx=150, min_ctx=40, spare_blocks=2)
    bm, k_pool, v_pool = setup(w)
    bs, Hkv = w.block_size, w.num_kv_heads
    q = workloads.draw_queries(w, 4, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, [0, 1, 2, 3])
    k0, v0 = to_f64(k_pool), to_f64(v_pool)
    before = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=32)
    check_close(to_f64(before), oracle.paged_decode(to_f64(q), k0, v0, tables, ctx_np, w.scale),
                dtype, "before swap")
    # the batch decoded after the swap-in (sequences 1..3), on the old placement
    before_123 = binding.decode_split(q[1:], k_pool, v_pool, bt[1:].contiguous(), ctx[1:].contiguous(),
                                      w.scale, partition_tokens=32)

    # preempt sequence 1: copy its blocks to host slots 0..n-1
    old = bm.swap_out(1)
    n = len(old)
    host_k = torch.empty((n,) + tuple(k_pool.shape[1:]), dtype=k_pool.dtype).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    out_pairs = torch.tensor([[b, i] for i, b in enumerate(old)], dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.swap_out(k_pool, v_pool, host_k, host_v, out_pairs, dev_err=err)
    torch.cuda.synchronize()
    # the host copies hold every slot of the sequence's blocks: the oracle's
    # gather through its old table over the pool equals its gather through
    # host slots 0..n-1 over the host buffers, bit for bit
    hk, hv = to_f64(host_k), to_f64(host_v)
    for kvh in range(Hkv):
        for pool, host in ((k0, hk), (v0, hv)):
            assert np.array_equal(oracle.gather_sequence(host, list(range(n)), n * bs, kvh),
                                  oracle.gather_sequence(pool, old, n * bs, kvh))

    # the pool reuses the reclaimed blocks: another sequence overwrites them
    bm.allocate(10, n * 16)
    reused = torch.tensor(bm.block_table(10), device="cuda")
    k_pool[reused] = torch.randn_like(k_pool[reused].float()).to(k_pool.dtype)
    v_pool[reused] = torch.randn_like(v_pool[reused].float()).to(v_pool.dtype)
    bm.free(0)                                   # room for the swap-in
    new = bm.swap_in(1)
    assert len(new) == n and set(new).isdisjoint(set(bm.block_table(10)))
    in_pairs = torch.tensor([[i, b] for i, b in enumerate(new)], dtype=torch.int64, device="cuda")
    binding.swap_in(host_k, host_v, k_pool, v_pool, in_pairs, dev_err=err)

    bt2, ctx2, tables2, ctx2_np = device_tables(bm, [1, 2, 3])
    after = binding.decode_split(q[1:], k_pool, v_pool, bt2, ctx2, w.scale, partition_tokens=32)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    k1, v1 = to_f64(k_pool), to_f64(v_pool)
    # the swapped-in blocks hold the host copies, bit for bit
    for kvh in range(Hkv):
        for pool, host in ((k1, hk), (v1, hv)):
            assert np.array_equal(oracle.gather_sequence(pool, new, n * bs, kvh),
                                  oracle.gather_sequence(host, list(range(n)), n * bs, kvh))
    check_close(to_f64(after), oracle.paged_decode(to_f64(q[1:]), k1, v1, tables2, ctx2_np, w.scale),
                dtype, "after swap-in")
    # placement does not matter: the same batch gives the same result as
    # before the swap, bit for bit
    assert torch.equal(after, before_123)


def test_swap_rejects_pageable_host_memory():
    k = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device="cuda")
    host = torch.zeros(2, 2, 16, 128, dtype=torch.bfloat16)      # not pinned
    pairs = torch.tensor([[0, 0]], dtype=torch.int64, device="cuda")
    with pytest.raises(binding.InvalidArgumentError):
        binding.swap_out(k, k, host, host, pairs)
