"""pa_prefill (causal chunked prefill over the paged cache) against the
oracle: batches mixing new-prompt prefill (no prior context), chunked
prefill on top of earlier context, single new tokens; query tiles that span
several KV partitions (partials + merge) and ones that fit one; GQA groups
1, 4, 8 and 16; head_dim 64 and 128; block sizes 16 and 32. Both prefill
kernels are covered: the tcgen05 one (default) and the mma.sync one
(PAGEDKV_PREFILL_KERNEL=mma_sync)."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu


# "tcgen05_3ctas": the tcgen05 kernel's persistent launch capped at 3 CTAs,
# so that every CTA runs many items back to back (idle second tiles, empty
# spans, partial last chunks and partition items in one CTA's sequence).
# "tcgen05_halves" / "tcgen05_halves_3ctas": the tcgen05 kernel with two
# softmax threads per query row (PAGEDKV_PREFILL_HALVES=2), full grid and
# capped at 3 CTAs.
KERNELS = ["tcgen05", "tcgen05_3ctas", "tcgen05_halves", "tcgen05_halves_3ctas", "mma_sync"]


@pytest.fixture(params=KERNELS)
def kernel(request, monkeypatch):
    if request.param == "mma_sync":
        monkeypatch.setenv("PAGEDKV_PREFILL_KERNEL", "mma_sync")
    else:
        monkeypatch.delenv("PAGEDKV_PREFILL_KERNEL", raising=False)
    if request.param.endswith("_3ctas"):
        monkeypatch.setenv("PAGEDKV_PREFILL_CTAS", "3")
    else:
        monkeypatch.delenv("PAGEDKV_PREFILL_CTAS", raising=False)
    if request.param.startswith("tcgen05_halves"):
        monkeypatch.setenv("PAGEDKV_PREFILL_HALVES", "2")
    else:
        monkeypatch.delenv("PAGEDKV_PREFILL_HALVES", raising=False)
    return request.param


@pytest.mark.parametrize("G,bs,partition,D", [(1, 16, 64, 128), (4, 16, 32, 128), (8, 32, 64, 128),
                                              (4, 32, 4096, 128), (16, 16, 128, 128),
                                              (2, 16, 64, 64), (8, 32, 4096, 64),
                                              # groups that do not divide a 128-row tile
                                              (6, 16, 64, 128), (3, 32, 4096, 64)])
def test_prefill_matches_oracle(kernel, G, bs, partition, D):
    # (context length, new tokens): prompt, chunk on prior context, single token, odd sizes
    plan = [(75, 75), (300, 37), (129, 1), (64, 64), (500, 130), (17, 9)]
    ctx = np.array([c for c, _ in plan], dtype=np.int64)
    qlen = np.array([n for _, n in plan], dtype=np.int32)
    w = workloads.random_small(71 + G, num_seqs=len(plan), num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=D, block_size=bs, dtype=workloads.BF16,
                               max_ctx=int(ctx.max()), fixed_lens=ctx.tolist())
    bm, k_pool, v_pool = setup(w)
    bt, ctx_d, tables, ctx_np = device_tables(bm, list(range(len(plan))))
    total = int(qlen.sum())
    q = workloads.draw_normal((total, 2 * G, D), workloads.BF16, 77, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, partition_tokens=partition,
                          dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, qlen,
                                w.scale)
    check_close(to_f64(out), want, workloads.BF16,
                f"prefill[{kernel}] G={G} bs={bs} part={partition} D={D}")


def _ramp_keys(k_pool, tables, ctx_np, amplitude):
    """Overwrite every key of every sequence with amplitude * t / ctx in all
    dimensions (t = the token's position): with all-ones queries each logit
    grows with t, so the running max rises at every KV chunk."""
    bs = k_pool.shape[2]
    for s, c in enumerate(ctx_np):
        c = int(c)
        for t in range(c):
            k_pool[int(tables[s, t // bs]), :, t % bs, :] = amplitude * t / c


def test_prefill_rising_logits(kernel):
    """Logits that grow along the context (the max moves in every chunk) and
    span many powers of two: exercises the rescaling of the accumulator."""
    G, bs, D = 4, 16, 128
    plan = [(700, 700), (450, 200), (64, 64)]
    ctx = np.array([c for c, _ in plan], dtype=np.int64)
    qlen = np.array([n for _, n in plan], dtype=np.int32)
    w = workloads.random_small(90, num_seqs=len(plan), num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=D, block_size=bs, dtype=workloads.BF16,
                               max_ctx=int(ctx.max()), fixed_lens=ctx.tolist())
    bm, k_pool, v_pool = setup(w)
    bt, _, tables, ctx_np = device_tables(bm, list(range(len(plan))))
    _ramp_keys(k_pool, tables, ctx_np, 3.0)  # logits from 0 to ~34 (~49 powers of two)
    total = int(qlen.sum())
    q = torch.ones((total, 2 * G, D), dtype=torch.bfloat16, device="cuda")
    want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, qlen,
                                w.scale)
    for partition in (64, 4096):
        out = binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale,
                              partition_tokens=partition)
        check_close(to_f64(out), want, workloads.BF16, f"rising[{kernel}] part={partition}")


def test_prefill_long_prompt(kernel):
    """One long prompt (many KV chunks per tile: the stage ring wraps many
    times) next to short ones, whole-context partitions."""
    G, bs, D = 2, 32, 128
    plan = [(1500, 1500), (40, 40), (1000, 3)]
    ctx = np.array([c for c, _ in plan], dtype=np.int64)
    qlen = np.array([n for _, n in plan], dtype=np.int32)
    w = workloads.random_small(91, num_seqs=len(plan), num_q_heads=G, num_kv_heads=1,
                               head_dim=D, block_size=bs, dtype=workloads.BF16,
                               max_ctx=int(ctx.max()), fixed_lens=ctx.tolist())
    bm, k_pool, v_pool = setup(w)
    bt, _, tables, ctx_np = device_tables(bm, list(range(len(plan))))
    total = int(qlen.sum())
    q = workloads.draw_normal((total, G, D), workloads.BF16, 92, "cuda")
    out = binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, partition_tokens=8192)
    want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, qlen,
                                w.scale)
    check_close(to_f64(out), want, workloads.BF16, f"long prompt[{kernel}]")


_FULL_SIZE_WANT = {}


def test_prefill_full_size(kernel):
    """The measured prefill configuration (16 sequences x (1024 prior + 1024
    new tokens), 32 query / 8 KV heads, head_dim 128, block 16, 512-token
    partitions): every (token, head) output against the oracle's causal
    prefill (evaluated once, shared by both kernels)."""
    B, prior, chunk, Hq, Hkv, D, bs = 16, 1024, 1024, 32, 8, 128, 16
    ctx = np.full(B, prior + chunk, dtype=np.int64)
    w = workloads.random_small(500, num_seqs=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=workloads.BF16, max_ctx=prior + chunk,
                               fixed_lens=ctx.tolist())
    bm, k_pool, v_pool = setup(w)
    bt, _, tables, ctx_np = device_tables(bm, list(range(B)))
    qlen = np.full(B, chunk, dtype=np.int32)
    q = workloads.draw_normal((B * chunk, Hq, D), workloads.BF16, 501, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, partition_tokens=512,
                          dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    if "want" not in _FULL_SIZE_WANT:
        _FULL_SIZE_WANT["want"] = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool),
                                                       tables, ctx_np, qlen, w.scale)
    check_close(to_f64(out), _FULL_SIZE_WANT["want"], workloads.BF16, f"full-size prefill[{kernel}]")


def test_prefill_of_one_token_equals_decode():
    w = workloads.random_small(80, num_seqs=5, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=600, min_ctx=1)
    bm, k_pool, v_pool = setup(w)
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(5)))
    q = workloads.draw_queries(w, 5, device="cuda")
    a = binding.prefill(q, k_pool, v_pool, bt, ctx_np, np.ones(5, np.int32), w.scale,
                        partition_tokens=64)
    b = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=64)
    check_close(to_f64(a), to_f64(b), workloads.BF16, "prefill(1) vs decode")


def test_prefill_rejects_bad_lengths():
    k = torch.zeros(8, 2, 16, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(5, 4, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(2, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(binding.InvalidArgumentError):
        binding.prefill(q, k, k, bt, [10, 3], [2, 4], 0.1)        # query_len > context_len
    with pytest.raises(binding.InvalidArgumentError):
        binding.prefill(q, k, k, bt, [10, 30], [2, 2], 0.1)       # sum of query_lens != 5


def test_prefill_with_empty_sequences(kernel):
    """Sequences with earlier context but no new tokens (query_len 0) sit in
    the batch beside ordinary ones; a batch with no new tokens at all
    returns at once."""
    G, bs, D = 4, 16, 128
    plan = [(90, 0), (200, 33), (0, 0), (47, 47), (130, 0)]
    ctx = np.array([c for c, _ in plan], dtype=np.int64)
    qlen = np.array([n for _, n in plan], dtype=np.int32)
    w = workloads.random_small(95, num_seqs=len(plan), num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=D, block_size=bs, dtype=workloads.BF16,
                               max_ctx=int(ctx.max()), fixed_lens=ctx.tolist())
    bm, k_pool, v_pool = setup(w)
    bt, _, tables, ctx_np = device_tables(bm, list(range(len(plan))))
    total = int(qlen.sum())
    q = workloads.draw_normal((total, 2 * G, D), workloads.BF16, 96, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, partition_tokens=64,
                          dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, qlen,
                                w.scale)
    check_close(to_f64(out), want, workloads.BF16, f"empty sequences[{kernel}]")
    q0 = torch.empty((0, 2 * G, D), dtype=torch.bfloat16, device="cuda")
    out0 = binding.prefill(q0, k_pool, v_pool, bt, ctx_np, np.zeros(len(plan), np.int32), w.scale,
                           partition_tokens=64)
    assert out0.shape == (0, 2 * G, D)
