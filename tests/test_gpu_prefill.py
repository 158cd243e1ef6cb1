"""pa_prefill (causal chunked prefill over the paged cache) against the
oracle: batches mixing new-prompt prefill (no prior context), chunked
prefill on top of earlier context, single new tokens; query tiles that span
several KV partitions (partials + merge) and ones that fit one; GQA groups
1, 4 and 8; block sizes 16 and 32."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,bs,partition", [(1, 16, 64), (4, 16, 32), (8, 32, 64), (4, 32, 4096)])
def test_prefill_matches_oracle(G, bs, partition):
    rng = np.random.default_rng(70 + G + bs)
    # (context length, new tokens): prompt, chunk on prior context, single token, odd sizes
    plan = [(75, 75), (300, 37), (129, 1), (64, 64), (500, 130), (17, 9)]
    ctx = np.array([c for c, _ in plan], dtype=np.int64)
    qlen = np.array([n for _, n in plan], dtype=np.int32)
    w = workloads.random_small(71 + G, num_seqs=len(plan), num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=128, block_size=bs, dtype=workloads.BF16,
                               max_ctx=int(ctx.max()), fixed_lens=ctx.tolist())
    bm, k_pool, v_pool = setup(w)
    bt, ctx_d, tables, ctx_np = device_tables(bm, list(range(len(plan))))
    total = int(qlen.sum())
    q = workloads.draw_normal((total, 2 * G, 128), workloads.BF16, 77, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, partition_tokens=partition,
                          dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, qlen,
                                w.scale)
    check_close(to_f64(out), want, workloads.BF16, f"prefill G={G} bs={bs} part={partition}")


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
