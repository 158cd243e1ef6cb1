"""pa_decode_split_window (sliding-window decode) against the oracle's
windowed definition: ragged contexts, windows shorter and longer than a
block or a partition, fp32 and bf16, MHA and GQA, block sizes 16 and 32,
head_dim 64, 128 and 256, and tables whose blocks before the window were
released (-1 entries)."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, device_tables, setup, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,G,bs", [(workloads.F32, 1, 16), (workloads.BF16, 1, 32),
                                        (workloads.BF16, 8, 16), (workloads.F32, 2, 32)])
@pytest.mark.parametrize("window", [1, 7, 16, 40, 97, 10_000])
@pytest.mark.parametrize("split_kernel", ["ticket", "stream"])
def test_window_matches_oracle(monkeypatch, split_kernel, dtype, G, bs, window):
    monkeypatch.setenv("PAGEDKV_SPLIT_KERNEL", split_kernel)
    w = workloads.random_small(60 + G + bs, num_seqs=7, num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=128, block_size=bs, dtype=dtype, max_ctx=12 * bs,
                               fixed_lens=[0, 1, 12 * bs, bs + 1])
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 7, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(7)))
    want = oracle.paged_decode_window(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np,
                                      w.scale, window)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = binding.decode_split_window(q, k_pool, v_pool, bt, ctx, w.scale, window,
                                      partition_tokens=2 * bs, dev_err=err)
    check_close(to_f64(out), want, dtype, f"window {window}")
    # release the blocks wholly before each window: the kernel never reads them
    for s in range(7):
        bm.release_before(s, max(0, int(ctx_np[s]) - window))
    bt2, _, tables2, _ = device_tables(bm, list(range(7)))
    out2 = binding.decode_split_window(q, k_pool, v_pool, bt2, ctx, w.scale, window,
                                       partition_tokens=2 * bs, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(out, out2)


@pytest.mark.parametrize("head_dim", [64, 256])
@pytest.mark.parametrize("window", [7, 40])
@pytest.mark.parametrize("split_kernel", ["ticket", "stream"])
def test_window_other_head_dims(monkeypatch, split_kernel, window, head_dim):
    """The window start on the head_dim 64 and 256 instances of both split
    kernels (bf16, GQA group 4, block 16), against the oracle."""
    monkeypatch.setenv("PAGEDKV_SPLIT_KERNEL", split_kernel)
    w = workloads.random_small(90 + head_dim, num_seqs=5, num_q_heads=8, num_kv_heads=2,
                               head_dim=head_dim, block_size=16, dtype=workloads.BF16,
                               max_ctx=200, fixed_lens=[0, 1, 200, 17])
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 5, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(5)))
    want = oracle.paged_decode_window(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np,
                                      w.scale, window)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = binding.decode_split_window(q, k_pool, v_pool, bt, ctx, w.scale, window,
                                      partition_tokens=32, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_close(to_f64(out), want, workloads.BF16, f"window {window}, head_dim {head_dim}")
