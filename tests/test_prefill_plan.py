"""pa_prefill_plan (host only, no GPU): the work plan of the tcgen05 prefill
kernel. Every (query token, KV head) pair is covered once per KV partition
of its causal span; each sequence's query runs come last-first; a
persistent schedule lists each CTA's items together in list order, uses
every item once, and keeps the CTAs' work close to even."""

import numpy as np
import pytest

from paged_kv_cache_336_b200 import binding

SEQ, QBEGIN, QCOUNT, KVH, PART, CTA = range(6)


def _batch(seed, n=6, max_ctx=700):
    rng = np.random.default_rng(seed)
    ctx = rng.integers(1, max_ctx, size=n)
    qlen = np.minimum(ctx, rng.integers(0, max_ctx, size=n))
    qlen[rng.random(n) < 0.2] = 0            # sequences with no new tokens
    qlen[rng.random(n) < 0.2] = 1            # single new tokens
    return ctx.astype(np.int32), qlen.astype(np.int32)


@pytest.mark.parametrize("G", [1, 2, 4, 6, 8, 16])
@pytest.mark.parametrize("bs,partition", [(16, 16), (16, 64), (32, 256), (16, 4096)])
def test_plan_covers_each_query_token_and_head_once_per_partition(G, bs, partition):
    Hkv = 2
    for seed in range(4):
        ctx, qlen = _batch(100 * G + seed)
        items, grid = binding.prefill_plan(ctx, qlen, G * Hkv, Hkv, bs, partition)
        assert grid == len(items)
        tq = 2 * max(1, 128 // G)            # query tokens per item: two 128-row tiles
        q_base = np.concatenate([[0], np.cumsum(qlen)[:-1]])
        seen = {}
        for row in items:
            s = int(row[SEQ])
            first = int(row[QBEGIN]) - int(q_base[s])   # run start within the sequence
            count = int(row[QCOUNT])
            assert first % tq == 0 and 0 < count <= tq and first + count <= qlen[s]
            assert count == min(tq, qlen[s] - first)
            key = (s, first, int(row[KVH]), int(row[PART]))
            assert key not in seen, f"duplicate item {key}"
            seen[key] = count
        for s in range(len(ctx)):
            for first in range(0, int(qlen[s]), tq):
                count = min(tq, int(qlen[s]) - first)
                kv_end = int(ctx[s]) - int(qlen[s]) + first + count   # last position + 1
                parts = -(-(-(-kv_end // bs)) // (partition // bs))
                for h in range(Hkv):
                    for p in range(parts):
                        assert seen.pop((s, first, h, p), None) == count, (s, first, h, p)
        assert not seen, f"items beyond the causal spans: {sorted(seen)[:4]}"


def test_plan_orders_each_sequences_runs_last_first():
    ctx, qlen = _batch(7, n=8, max_ctx=2000)
    items, _ = binding.prefill_plan(ctx, qlen, 32, 8, 16, 512)
    seqs = items[:, SEQ]
    assert np.all(np.diff(seqs) >= 0), "sequence order"
    for s in np.unique(seqs):
        starts = items[seqs == s, QBEGIN]
        runs = starts[np.r_[True, np.diff(starts) != 0]]
        assert np.all(np.diff(runs) < 0), f"sequence {s}: runs not last-first"


def _span(row, ctx, qlen, q_base, bs, partition):
    """KV tokens the item reads: its partition of [0, last position + 1)."""
    s = int(row[SEQ])
    kv_end = int(ctx[s]) - int(qlen[s]) + int(row[QBEGIN]) - int(q_base[s]) + int(row[QCOUNT])
    lo = int(row[PART]) * partition
    return max(0, min(kv_end, lo + partition) - lo)


@pytest.mark.parametrize("ctas", [3, 17, 148])
def test_schedule_lists_each_ctas_items_in_order_and_balances_them(ctas):
    ctx = np.full(16, 2048, np.int32)
    qlen = np.full(16, 1024, np.int32)
    plain, _ = binding.prefill_plan(ctx, qlen, 32, 8, 16, 2048)
    sched, grid = binding.prefill_plan(ctx, qlen, 32, 8, 16, 2048, max_ctas=ctas)
    assert grid == ctas and len(sched) == len(plain) == 2048
    cta = sched[:, CTA]
    assert cta.min() == 0 and cta.max() == ctas - 1
    assert np.all(np.diff(cta) >= 0), "items listed CTA by CTA"
    # every item once; within a CTA, in the unscheduled list order
    pos = {tuple(r[:5]): i for i, r in enumerate(plain)}
    idx = np.array([pos[tuple(r[:5])] for r in sched])
    assert sorted(idx.tolist()) == list(range(len(plain)))
    for b in range(ctas):
        assert np.all(np.diff(idx[cta == b]) > 0), f"CTA {b}: items out of list order"
    # list scheduling to the least-loaded CTA: no CTA ends more than one item
    # (the largest span, 2048 KV tokens here) above the mean
    q_base = np.concatenate([[0], np.cumsum(qlen)[:-1]])
    spans = np.array([_span(r, ctx, qlen, q_base, 16, 2048) for r in sched])
    load = np.bincount(cta, weights=spans, minlength=ctas)
    assert load.max() <= load.mean() + spans.max(), (load.max(), load.mean(), spans.max())


def test_schedule_only_when_items_exceed_the_ctas():
    ctx, qlen = _batch(3)
    plain, n = binding.prefill_plan(ctx, qlen, 8, 2, 16, 64)
    same, grid = binding.prefill_plan(ctx, qlen, 8, 2, 16, 64, max_ctas=n)
    assert grid == n and np.array_equal(plain, same)
    assert np.array_equal(plain[:, CTA], np.arange(n))


def test_empty_batch_and_no_new_tokens():
    items, grid = binding.prefill_plan(np.array([5, 9], np.int32), np.array([0, 0], np.int32),
                                       4, 4, 16, 64, max_ctas=2)
    assert items.shape == (0, 6) and grid == 0


def test_plan_rejects_bad_arguments():
    ctx, qlen = np.array([40], np.int32), np.array([8], np.int32)
    with pytest.raises(binding.PagedKVError) as e:
        binding.prefill_plan(ctx, qlen, 4, 4, 8, 64)            # block size 8
    assert e.value.status == binding.PA_ERR_UNSUPPORTED
    for bad in [dict(partition_tokens=40), dict(num_q_heads=6, num_kv_heads=4)]:
        kw = dict(num_q_heads=4, num_kv_heads=4, block_size=16, partition_tokens=64)
        kw.update(bad)
        with pytest.raises(binding.InvalidArgumentError):
            binding.prefill_plan(ctx, qlen, **kw)
    with pytest.raises(binding.InvalidArgumentError):
        binding.prefill_plan(np.array([4], np.int32), np.array([5], np.int32), 4, 4, 16, 64)
