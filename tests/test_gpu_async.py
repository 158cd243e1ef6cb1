"""Calls that build a plan on the host (pa_prefill, pa_decode_shared_prefix)
enqueue their work and return without waiting for the stream.

Small plans go up as the parameters of a scatter kernel; larger ones (or
all, with PAGEDKV_PLAN_UPLOAD=staging) from the library's page-locked
staging ring. Either way a call issued behind a long-running kernel returns
while that kernel still runs. Back-to-back calls behind a ~0.5 s spin kernel
must all return in a small fraction of it, with the stream still busy
afterwards, and their results must still match the oracle. Both upload
paths are run.
"""

import time

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("prefix_kernel", ["mma_sync", "tcgen05"])
@pytest.mark.parametrize("upload", ["params", "staging"])
def test_plan_uploads_do_not_wait_for_the_stream(monkeypatch, upload, prefix_kernel):
    # staging + tcgen05: the prefix plan's pieces lie far apart in the
    # workspace (items, then the Q-tile list), so they go up as two copies
    if upload == "staging":
        monkeypatch.setenv("PAGEDKV_PLAN_UPLOAD", "staging")
    if prefix_kernel == "tcgen05":
        monkeypatch.setenv("PAGEDKV_PREFIX_KERNEL", "tcgen05")
    w = workloads.random_small(31, num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=160,
                               fixed_lens=[160, 70, 20])
    bm, k_pool, v_pool = setup(w)
    bt, _, tables, ctx_np = device_tables(bm, [0, 1, 2])
    qlen = np.array([160, 30, 5], dtype=np.int32)
    q = workloads.draw_normal((int(qlen.sum()), 8, 128), workloads.BF16, 32, "cuda")
    ws = binding.prefill_workspace(3, int(qlen.sum()), 8, 2, 128, 16, w.max_blocks_per_seq, 64)
    outs = [torch.empty_like(q) for _ in range(6)]

    # shared-prefix inputs: one prompt forked into 4 branches
    NB = 64
    sbm = binding.BlockManager(NB, 16, 16, np.arange(NB, dtype=np.int32))
    sbm.allocate(0, 70)
    for c in (1, 2, 3):
        sbm.fork(0, c)
    sw = workloads.random_small(33, num_seqs=1, num_q_heads=8, num_kv_heads=2, head_dim=128,
                                block_size=16, dtype=workloads.BF16, max_ctx=1)
    sw.num_blocks = NB
    sk, sv = workloads.draw_pools(sw, "cuda")
    sq = workloads.draw_queries(sw, 4, device="cuda")
    sbt, sctx, stables, sctx_np = device_tables(sbm, [0, 1, 2, 3])
    groups = sbm.prefix_groups([0, 1, 2, 3])
    sws = binding.shared_prefix_workspace(4, 8, 2, 128, 16, 16, 32)
    souts = [torch.empty_like(sq) for _ in range(6)]

    def calls(i):
        binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, partition_tokens=64,
                        out=outs[i], workspace=ws)
        binding.decode_shared_prefix(sq, sk, sv, sbt, sctx, sw.scale, groups, partition_tokens=32,
                                     out=souts[i], workspace=sws)

    calls(0)                       # warm-up: kernels prepared, staging ring allocated
    torch.cuda.synchronize()
    torch.cuda._sleep(1_000_000_000)   # ~0.5 s of spinning on the stream
    t0 = time.perf_counter()
    for i in range(1, 6):
        calls(i)
    host_s = time.perf_counter() - t0
    still_busy = not torch.cuda.current_stream().query()
    torch.cuda.synchronize()
    assert still_busy, "the calls waited for the stream"
    assert host_s < 0.1, f"10 calls took {host_s:.3f} s of host time"

    want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, qlen,
                                w.scale)
    swant = oracle.paged_decode(to_f64(sq), to_f64(sk), to_f64(sv), stables, sctx_np, sw.scale)
    for i in range(6):
        check_close(to_f64(outs[i]), want, workloads.BF16, f"prefill call {i}")
        check_close(to_f64(souts[i]), swant, workloads.BF16, f"shared prefix call {i}")
