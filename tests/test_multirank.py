"""Multi-process host logic on CPU (gloo, world size 2).

The decode path partitions by sequence: every rank owns its batch, its pool
and its own block manager, and no data crosses ranks. What does cross is the
measurement: the job time is the slowest rank's and the bytes/tokens are
summed. These tests run that reduction and the per-rank workload setup in two
gloo processes.
"""

import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world))
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
        import bench
        from paged_kv_cache_336_b200.binding import BlockManager
        w = bench.make_workload("gqa", rank)
        bm = BlockManager(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
        for s in w.prefill_seqs:
            bm.allocate(s, int(w.context_lens[s]))
        slots, pairs = bm.append_slots_arrays(w.step_seqs)
        tables, ctx = bm.export(w.decode_seqs)
        local_bytes = bench.decode_bytes(w, ctx.astype(np.int64))
        local_ms = 10.0 + 3.0 * rank
        red = bench.reduce_over_ranks(local_ms, local_bytes, len(ctx), torch.device("cpu"))
        gathered = [None] * world
        dist.all_gather_object(gathered, (int(ctx.sum()), int(tables[0, 0]), local_bytes))
        dist.barrier()
        dist.destroy_process_group()
        out_q.put((rank, red, gathered, None))
    except Exception as e:  # report instead of hanging the parent
        out_q.put((rank, None, None, repr(e)))


def test_two_ranks_reduce_time_max_and_bytes_sum():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            rank, red, gathered, err = q.get(timeout=120)
            assert err is None, f"rank {rank}: {err}"
            results[rank] = (red, gathered)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    assert set(results) == {0, 1}
    (red0, g0), (red1, g1) = results[0], results[1]
    assert red0 == red1                      # every rank sees the same job figures
    ms, total_bytes, tokens = red0
    assert ms == 13.0                        # slowest rank
    assert total_bytes == g0[0][2] + g0[1][2]
    assert tokens == 512                     # 256 sequences per rank
    assert g0[0][:2] != g0[1][:2]            # ranks run different batches (seeded by rank)


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    assert bench.reduce_over_ranks(1.5, 100, 7, torch.device("cpu")) == (1.5, 100.0, 7.0)
