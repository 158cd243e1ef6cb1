"""Guard bands around output buffers: every decode and prefill entry point
writes its output and nothing next to it.

Each output lives in the middle of a larger device buffer whose bytes are
first set to a sentinel; after the call the bytes before and after the
output must still hold it, and the output itself must match the float64
oracle (so every element in between was written). Covered: pa_decode,
pa_decode_split, pa_decode_split_static, pa_decode_shared_prefix,
pa_decode_split_window and pa_prefill, on ragged batches with empty and
one-token sequences, MHA and GQA.
"""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu

PAD = 4096          # guard bytes on each side
SENTINEL = 0xA5


def guarded_like(t: torch.Tensor):
    """(raw buffer, view shaped like t) with PAD sentinel bytes on each side."""
    n = t.numel() * t.element_size()
    raw = torch.full((2 * PAD + n,), SENTINEL, dtype=torch.uint8, device=t.device)
    out = raw[PAD:PAD + n].view(t.dtype).view(t.shape)
    return raw, out


def assert_guards_intact(raw: torch.Tensor, what: str):
    torch.cuda.synchronize()
    n = raw.numel() - 2 * PAD
    assert torch.all(raw[:PAD] == SENTINEL), f"{what}: bytes before the output were written"
    assert torch.all(raw[PAD + n:] == SENTINEL), f"{what}: bytes after the output were written"


def _small(dtype, G, seed=70):
    w = workloads.random_small(seed + G, num_seqs=6, num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=128, block_size=16, dtype=dtype, max_ctx=300,
                               fixed_lens=[0, 1, 300])
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 6, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(6)))
    want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, w.scale)
    return w, bm, k_pool, v_pool, q, bt, ctx, tables, ctx_np, want


@pytest.mark.parametrize("dtype,G", [(workloads.F32, 1), (workloads.BF16, 1), (workloads.BF16, 8)])
@pytest.mark.parametrize("split_kernel", ["ticket", "stream"])
def test_decode_entry_points_write_only_their_output(monkeypatch, split_kernel, dtype, G):
    monkeypatch.setenv("PAGEDKV_SPLIT_KERNEL", split_kernel)
    w, bm, k_pool, v_pool, q, bt, ctx, tables, ctx_np, want = _small(dtype, G)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    raw, out = guarded_like(q)
    binding.decode(q, k_pool, v_pool, bt, ctx, w.scale, out=out, dev_err=err)
    assert_guards_intact(raw, "pa_decode")
    check_close(to_f64(out), want, dtype, "pa_decode")

    raw, out = guarded_like(q)
    binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=32, out=out,
                         dev_err=err)
    assert_guards_intact(raw, "pa_decode_split")
    check_close(to_f64(out), want, dtype, "pa_decode_split")

    raw, out = guarded_like(q)
    lib = binding.library()
    dt = binding.PA_F32 if q.dtype == torch.float32 else binding.PA_BF16
    st = lib.pa_decode_split_static(
        q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), bt.data_ptr(), ctx.data_ptr(), 6,
        2 * G, 2, 128, 16, w.num_blocks, bt.shape[1], float(w.scale), dt, 32, out.data_ptr(),
        err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == binding.PA_OK, lib.pa_last_error_string()
    assert_guards_intact(raw, "pa_decode_split_static")
    check_close(to_f64(out), want, dtype, "pa_decode_split_static")

    window = 40
    want_w = oracle.paged_decode_window(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np,
                                        w.scale, window)
    raw, out = guarded_like(q)
    binding.decode_split_window(q, k_pool, v_pool, bt, ctx, w.scale, window, partition_tokens=32,
                                out=out, dev_err=err)
    assert_guards_intact(raw, "pa_decode_split_window")
    check_close(to_f64(out), want_w, dtype, "pa_decode_split_window")
    torch.cuda.synchronize()
    assert int(err.item()) == 0


@pytest.mark.parametrize("G", [1, 4])
@pytest.mark.parametrize("split_kernel", ["ticket", "stream"])
def test_shared_prefix_writes_only_its_output(monkeypatch, split_kernel, G):
    monkeypatch.setenv("PAGEDKV_SPLIT_KERNEL", split_kernel)
    bs, Hkv, D = 16, 2, 128
    rng = np.random.default_rng(5 + G)
    NB = 200
    bm = binding.BlockManager(NB, bs, 32, rng.permutation(NB).astype(np.int32))
    bm.allocate(0, 5 * bs + 3)
    seqs = [0]
    for c in range(1, 6):
        bm.fork(0, c)
        seqs.append(c)
    for s in seqs:
        for _ in range(int(rng.integers(0, 20))):
            bm.append_slot(s)
    bm.allocate(9, 0)
    seqs.append(9)
    w = workloads.random_small(8, num_seqs=1, num_q_heads=G * Hkv, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=workloads.BF16, max_ctx=1)
    w.num_blocks = NB
    k_pool, v_pool = workloads.draw_pools(w, "cuda")
    q = workloads.draw_queries(w, len(seqs), device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, seqs)
    groups = bm.prefix_groups(seqs)
    raw, out = guarded_like(q)
    binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups, partition_tokens=32,
                                 out=out)
    assert_guards_intact(raw, "pa_decode_shared_prefix")
    want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, w.scale)
    check_close(to_f64(out), want, w.dtype, "pa_decode_shared_prefix")


@pytest.mark.parametrize("partition", [64, 4096])
def test_prefill_writes_only_its_output(partition):
    w = workloads.random_small(12, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=200,
                               fixed_lens=[200, 97, 1, 33])
    bm, k_pool, v_pool = setup(w)
    bt, _, tables, ctx_np = device_tables(bm, list(range(4)))
    qlen = np.array([200, 30, 1, 0], dtype=np.int32)
    q = workloads.draw_normal((int(qlen.sum()), 8, 128), workloads.BF16, 13, "cuda")
    raw, out = guarded_like(q)
    binding.prefill(q, k_pool, v_pool, bt, ctx_np, qlen, w.scale, partition_tokens=partition,
                    out=out)
    assert_guards_intact(raw, "pa_prefill")
    want = oracle.paged_prefill(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, qlen,
                                w.scale)
    check_close(to_f64(out), want, workloads.BF16, "pa_prefill")
