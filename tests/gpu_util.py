"""Helpers shared by the GPU parity tests: workload setup on the device and
oracle evaluation of sampled outputs (the oracle runs on the CPU in float64)."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_336_b200 import workloads
from paged_kv_cache_336_b200.binding import BlockManager

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
F32_MAX_ABS = 1e-5


def build_tables(bm, w):
    for s in w.prefill_seqs:
        bm.allocate(s, int(w.context_lens[s]))
    for parent, child in w.forks:
        bm.fork(parent, child)
    for s, n in sorted(w.extra_tokens.items()):
        for _ in range(n):
            bm.append_slot(s)


def setup(w, device="cuda"):
    bm = BlockManager(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
    build_tables(bm, w)
    k_pool, v_pool = workloads.draw_pools(w, device)
    return bm, k_pool, v_pool


def device_tables(bm, seqs, device="cuda"):
    tables, ctx = bm.export(seqs, pad_value=-1)
    return (torch.from_numpy(tables).to(device), torch.from_numpy(ctx).to(device), tables, ctx)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_one(q, k_pool, v_pool, table_row, ctx, scale, s, h):
    """Oracle output of (s, h), copying to the host only the (block, KV head)
    tiles that query head reads; the oracle sees a one-KV-head pool holding
    those tiles in logical order and the query rows of that head's group."""
    _, Hkv, bs, D = k_pool.shape
    G = q.shape[1] // Hkv
    kvh = h // G
    nb = -(-int(ctx) // bs)
    blocks = torch.as_tensor(np.asarray(table_row[:nb], dtype=np.int64), device=k_pool.device)
    kp = to_f64(k_pool[:, kvh:kvh + 1].index_select(0, blocks)) if nb else np.zeros((0, 1, bs, D))
    vp = to_f64(v_pool[:, kvh:kvh + 1].index_select(0, blocks)) if nb else np.zeros((0, 1, bs, D))
    qs = to_f64(q[s:s + 1, kvh * G:(kvh + 1) * G])
    return oracle.paged_decode_one(qs, kp, vp, np.arange(max(nb, 1))[None, :], [int(ctx)], scale,
                                   0, h - kvh * G)


def check_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str = ""):
    err = np.abs(got - want)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if dtype == workloads.F32:
        assert err.max() <= F32_MAX_ABS, f"{what}: max abs err {err.max():.3e} > {F32_MAX_ABS}"
    else:
        assert err.max() <= BF16_MAX_ABS, f"{what}: max abs err {err.max():.3e} > {BF16_MAX_ABS}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e} > {BF16_MEAN_ABS}"
    return float(err.max()), float(err.mean())


def sample_pairs(rng, num_seqs, num_q_heads, n, must=()):
    pairs = set(must)
    while len(pairs) < min(n, num_seqs * num_q_heads):
        pairs.add((int(rng.integers(num_seqs)), int(rng.integers(num_q_heads))))
    return sorted(pairs)
