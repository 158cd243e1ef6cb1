"""Helpers shared by the GPU parity tests: workload setup on the device and
oracle evaluation of whole outputs (the oracle runs on the CPU in float64 and
walks the real block tables itself)."""

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


def host_slice(pool: torch.Tensor, kv_head: int, bits: bool = False) -> np.ndarray:
    """One KV head's slice of a device pool, ``[num_blocks, 1, block_size,
    head_dim]``, copied to the host: float32 values (bf16 widens exactly), or
    with ``bits`` the raw element bit patterns (int16 for bf16, int32 for
    fp32) for bit-exact comparisons. Physical block ids are unchanged, so the
    oracle walks the real block tables over it."""
    sl = pool[:, kv_head:kv_head + 1].contiguous()
    if bits:
        return sl.view(torch.int16 if pool.element_size() == 2 else torch.int32).cpu().numpy()
    return sl.float().cpu().numpy()


def as_bits(t: torch.Tensor) -> np.ndarray:
    """Raw element bit patterns of a device tensor, on the host."""
    t = t.contiguous()
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32).cpu().numpy()


def oracle_decode_by_kv_head(q, k_pool, v_pool, tables, ctx, scale) -> np.ndarray:
    """oracle.paged_decode over every (sequence, query head) of a batch whose
    pools are too large to copy to the host whole: one KV head at a time, the
    oracle gets that head's slice of both pools (``host_slice``), the query
    rows of its group and the real block tables and context lengths, and does
    its own gather through the tables. Returns float64 [B, Hq, D]."""
    B, Hq, D = q.shape
    Hkv = k_pool.shape[1]
    G = Hq // Hkv
    q64 = to_f64(q)
    out = np.empty((B, Hq, D), dtype=np.float64)
    for kvh in range(Hkv):
        kp = host_slice(k_pool, kvh)
        vp = host_slice(v_pool, kvh)
        out[:, kvh * G:(kvh + 1) * G] = oracle.paged_decode(q64[:, kvh * G:(kvh + 1) * G], kp, vp,
                                                            tables, ctx, scale)
        del kp, vp
    return out


def check_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str = ""):
    err = np.abs(got - want)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if dtype == workloads.F32:
        assert err.max() <= F32_MAX_ABS, f"{what}: max abs err {err.max():.3e} > {F32_MAX_ABS}"
    else:
        assert err.max() <= BF16_MAX_ABS, f"{what}: max abs err {err.max():.3e} > {BF16_MAX_ABS}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e} > {BF16_MEAN_ABS}"
    return float(err.max()), float(err.mean())


