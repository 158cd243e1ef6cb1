"""Host-planned calls inside CUDA graphs.

pa_decode_shared_prefix and pa_prefill build a plan on the host. A plan of
up to 30 KB reaches the device as the parameters of a scatter kernel, so the
call can be captured: the graph carries the plan, and each replay scatters
it again before the attention kernels run. These tests capture both calls,
replay them with new query values written into the captured buffers, and
compare every replay with the float64 oracle. A plan forced through the
staging ring (PAGEDKV_PLAN_UPLOAD=staging) must be refused during capture
with PA_ERR_UNSUPPORTED, and the same call must then run eagerly.
"""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu


def _shared_prefix_case(G=4):
    NB, bs, Hkv, D = 96, 16, 2, 128
    rng = np.random.default_rng(41)
    bm = binding.BlockManager(NB, bs, 24, rng.permutation(NB).astype(np.int32))
    bm.allocate(0, 5 * bs + 7)
    seqs = [0]
    for c in range(1, 6):
        bm.fork(0, c)
        seqs.append(c)
    for s in seqs:
        for _ in range(int(rng.integers(0, 25))):
            bm.append_slot(s)
    w = workloads.random_small(42, num_seqs=1, num_q_heads=G * Hkv, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=workloads.BF16, max_ctx=1)
    w.num_blocks = NB
    k_pool, v_pool = workloads.draw_pools(w, "cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, seqs)
    groups = bm.prefix_groups(seqs)
    return w, k_pool, v_pool, bt, ctx, tables, ctx_np, groups, len(seqs)


def test_shared_prefix_call_replays_from_a_graph():
    w, k_pool, v_pool, bt, ctx, tables, ctx_np, groups, B = _shared_prefix_case()
    q = workloads.draw_queries(w, B, device="cuda")
    out = torch.empty_like(q)
    ws = binding.shared_prefix_workspace(B, w.num_q_heads, w.num_kv_heads, w.head_dim, 16, 24, 32)
    binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups, partition_tokens=32,
                                 out=out, workspace=ws)   # eager first: kernels prepared
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups,
                                     partition_tokens=32, out=out, workspace=ws)
    for step in range(3):
        q.copy_(workloads.draw_queries(w, B, step=step + 1, device="cuda"))
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np,
                                   w.scale)
        check_close(to_f64(out), want, workloads.BF16, f"graph replay {step}")


def test_prefill_call_replays_from_a_graph():
    w = workloads.random_small(43, num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=200,
                               fixed_lens=[200, 90, 17])
    bm, k_pool, v_pool = setup(w)
    bt, _, tables, ctx_np = device_tables(bm, [0, 1, 2])
    qlen = np.array([120, 33, 1], dtype=np.int32)
    q = workloads.draw_normal((int(qlen.sum()), 8, 128), workloads.BF16, 44, "cuda")
    out = torch.empty_like(q)
    ws = binding.prefill_workspace(3, int(qlen.sum()), 8, 2, 128, 16, w.max_blocks_per_seq, 64)
    binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, 64, out, ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, 64, out, ws)
    for step in range(2):
        q.copy_(workloads.draw_normal(tuple(q.shape), workloads.BF16, 45 + step, "cuda"))
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np,
                                    qlen, w.scale)
        check_close(to_f64(out), want, workloads.BF16, f"prefill graph replay {step}")


def test_staged_plan_is_refused_during_capture(monkeypatch):
    w, k_pool, v_pool, bt, ctx, tables, ctx_np, groups, B = _shared_prefix_case()
    q = workloads.draw_queries(w, B, device="cuda")
    out = torch.empty_like(q)
    ws = binding.shared_prefix_workspace(B, w.num_q_heads, w.num_kv_heads, w.head_dim, 16, 24, 32)
    binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups, partition_tokens=32,
                                 out=out, workspace=ws)
    torch.cuda.synchronize()
    monkeypatch.setenv("PAGEDKV_PLAN_UPLOAD", "staging")
    g = torch.cuda.CUDAGraph()
    # torch warns that the captured graph is empty: the refusal came before
    # the call enqueued anything
    with pytest.warns(UserWarning, match="Graph is empty"):
        with pytest.raises(binding.PagedKVError) as info:
            with torch.cuda.graph(g):
                binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups,
                                             partition_tokens=32, out=out, workspace=ws)
    assert info.value.status == binding.PA_ERR_UNSUPPORTED
    assert "captured" in str(info.value)
    torch.cuda.synchronize()
    # the same call, eagerly, through the staging ring
    out.zero_()
    binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups, partition_tokens=32,
                                 out=out, workspace=ws)
    torch.cuda.synchronize()
    want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, w.scale)
    check_close(to_f64(out), want, workloads.BF16, "eager after refused capture")
