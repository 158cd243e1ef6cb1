"""GPU parity at the full sizes of the measured workloads, in the launch
configuration the bench times (block-manager step, copy-on-write copies,
append, split decode with 512-token partitions).

The oracle evaluates sampled (sequence, query head) outputs one by one
(always including the longest and shortest sequences); copies and appends
are checked bit-exactly on every block and slot they touch.
"""

import numpy as np
import pytest
import torch

from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, oracle_one, sample_pairs, setup, to_f64

pytestmark = pytest.mark.gpu


def _step_and_decode(w, n_samples, partition_tokens=512):
    bm, k_pool, v_pool = setup(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pairs = np.zeros((0, 2), dtype=np.int64)
    slots = np.zeros(0, dtype=np.int64)
    if w.step_seqs:
        slots, pairs = bm.append_slots_arrays(w.step_seqs)
        k_new, v_new = workloads.draw_new_kv(w, len(w.step_seqs), device="cuda")
        src_before_k = k_pool[torch.from_numpy(pairs[:, 0]).cuda()].clone() if len(pairs) else None
        if len(pairs):
            binding.copy_blocks(k_pool, v_pool, torch.from_numpy(pairs).cuda(), dev_err=err)
        binding.kv_append(k_new, v_new, torch.from_numpy(slots).cuda(), k_pool, v_pool, dev_err=err)
        torch.cuda.synchronize()
        # appended tokens landed bit-exactly
        sl = torch.from_numpy(slots).cuda()
        blk, off = sl // w.block_size, sl % w.block_size
        assert torch.equal(k_pool[blk, :, off, :], k_new)
        assert torch.equal(v_pool[blk, :, off, :], v_new)
        if len(pairs):
            # the copy holds the shared block's tokens; only the appended slot differs
            dst = torch.from_numpy(pairs[:, 1]).cuda()
            got = k_pool[dst].clone()
            for i, (s_dst) in enumerate(pairs[:, 1]):
                j = int(np.nonzero(slots // w.block_size == s_dst)[0][0])
                got[i, :, int(slots[j] % w.block_size), :] = src_before_k[i, :, int(slots[j] % w.block_size), :]
            assert torch.equal(got, src_before_k)
    seqs = w.decode_seqs
    bt, ctx, tables, ctx_np = device_tables(bm, seqs)
    q = workloads.draw_queries(w, len(seqs), device="cuda")
    out = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale,
                               partition_tokens=partition_tokens, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(w.seed)
    must = [(int(np.argmax(ctx_np)), 0), (int(np.argmin(ctx_np)), w.num_q_heads - 1)]
    got, want = [], []
    for s, h in sample_pairs(rng, len(seqs), w.num_q_heads, n_samples, must):
        want.append(oracle_one(q, k_pool, v_pool, tables[s], ctx_np[s], w.scale, s, h))
        got.append(to_f64(out[s, h]))
    return np.stack(got), np.stack(want), len(pairs)


def test_mha_batch64():
    w = workloads.mha()
    got, want, n_cow = _step_and_decode(w, 12)
    check_close(got, want, w.dtype, "mha")
    assert n_cow == 0


def test_gqa_batch256():
    w = workloads.gqa()
    got, want, _ = _step_and_decode(w, 12)
    check_close(got, want, w.dtype, "gqa")


def test_prefix_sharing():
    w = workloads.prefix()
    got, want, n_cow = _step_and_decode(w, 10)
    check_close(got, want, w.dtype, "prefix")


def test_prefix_sharing_cow_step():
    w = workloads.prefix_cow()
    got, want, n_cow = _step_and_decode(w, 10)
    check_close(got, want, w.dtype, "prefix_cow")
    assert n_cow == 120


@pytest.mark.parametrize("bs", [16, 32])
def test_long_context_split(bs):
    w = workloads.long(block_size=bs, slack=0.1)
    got, want, _ = _step_and_decode(w, 4)
    check_close(got, want, w.dtype, f"long bs{bs}")
