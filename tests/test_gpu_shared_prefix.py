"""pa_decode_shared_prefix against the oracle.

Forked sequences share their prompt's blocks; the shared-prefix route reads
them once per KV head for the whole group and must still return plain decode
attention. Small cases are compared with the full float64 oracle (several
groups, a group wider than one CTA's rows, sequences in no group, block
sizes 16 and 32, head_dim 128 and 64); the full-size prefix-sharing
workloads on every output row as well.
Both prefix-pass kernels are covered: the mma.sync one (default, 64 query
rows per CTA) and the tcgen05 one (PAGEDKV_PREFIX_KERNEL=tcgen05, 128).
"""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import (check_close, device_tables, oracle_decode_by_kv_head, setup, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["mma_sync", "tcgen05"])
def kernel(request, monkeypatch):
    if request.param == "tcgen05":
        monkeypatch.setenv("PAGEDKV_PREFIX_KERNEL", "tcgen05")
    else:
        monkeypatch.delenv("PAGEDKV_PREFIX_KERNEL", raising=False)
    return request.param


@pytest.mark.parametrize("G,bs,branches", [(1, 16, 5), (4, 16, 16), (8, 32, 12), (4, 32, 3),
                                           (16, 16, 20), (6, 32, 7)])
@pytest.mark.parametrize("split_kernel", ["ticket", "stream"])
def test_shared_prefix_small_matches_oracle(monkeypatch, kernel, split_kernel, G, bs, branches):
    _small_case(monkeypatch, split_kernel, G, bs, branches, 128)


@pytest.mark.parametrize("G,bs,branches", [(4, 16, 16), (8, 32, 12)])
@pytest.mark.parametrize("split_kernel", ["ticket", "stream"])
def test_shared_prefix_head_dim_64(monkeypatch, kernel, split_kernel, G, bs, branches):
    """The head_dim 64 instances of both prefix kernels and both suffix kernels."""
    _small_case(monkeypatch, split_kernel, G, bs, branches, 64)


def _small_case(monkeypatch, split_kernel, G, bs, branches, D):
    monkeypatch.setenv("PAGEDKV_SPLIT_KERNEL", split_kernel)
    Hkv = 2
    rng = np.random.default_rng(40 + G + bs)
    NB = 400
    bm = binding.BlockManager(NB, bs, 64, rng.permutation(NB).astype(np.int32))
    seqs = []
    nid = 0
    for prompt_len in (7 * bs + 3, 4 * bs, 2 * bs + 9):     # partial, exact, partial prompt tails
        root = nid
        bm.allocate(root, prompt_len)
        seqs.append(root)
        nid += 1
        for _ in range(branches - 1):
            bm.fork(root, nid)
            seqs.append(nid)
            nid += 1
    for s in seqs:                                            # private tokens (copy-on-write on the way)
        for _ in range(int(rng.integers(0, 2 * bs))):
            r = bm.append_slot(s)
    for extra in range(3):                                    # sequences in no group
        bm.allocate(nid, int(rng.integers(0, 6 * bs)))
        seqs.append(nid)
        nid += 1
    order = list(rng.permutation(seqs))
    w = workloads.random_small(7, num_seqs=1, num_q_heads=G * Hkv, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=workloads.BF16, max_ctx=1)
    w.num_blocks = NB
    k_pool, v_pool = workloads.draw_pools(w, "cuda")
    q = workloads.draw_queries(w, len(order), device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, order)
    groups = bm.prefix_groups(order)
    assert len(groups[2]) >= 2
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups,
                                       partition_tokens=2 * bs, dev_err=err)
    ref = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=2 * bs)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np, w.scale)
    check_close(to_f64(out), want, w.dtype, "shared prefix")
    check_close(to_f64(ref), want, w.dtype, "split")
    # twice in a row on the same workspace-less call path, and with no groups at all
    out2 = binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups,
                                        partition_tokens=2 * bs)
    assert torch.equal(out, out2)
    empty = (np.zeros(1, np.int32), np.zeros(0, np.int32), np.zeros(0, np.int32))
    out3 = binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, empty,
                                        partition_tokens=2 * bs)
    check_close(to_f64(out3), want, w.dtype, "no groups")


@pytest.mark.parametrize("name", ["prefix", "prefix_cow"])
def test_shared_prefix_full_size(monkeypatch, name):
    """Both prefix-pass kernels on the full-size workload after its append
    step; every output row against one oracle evaluation (the oracle walks
    the real tables over one KV head's pool slice at a time)."""
    w = workloads.WORKLOADS[name]()
    bm, k_pool, v_pool = setup(w)
    slots, pairs = bm.append_slots_arrays(w.step_seqs)
    kn, vn = workloads.draw_new_kv(w, len(w.step_seqs), device="cuda")
    if len(pairs):
        binding.copy_blocks(k_pool, v_pool, torch.from_numpy(pairs).cuda())
    binding.kv_append(kn, vn, torch.from_numpy(slots).cuda(), k_pool, v_pool)
    seqs = w.decode_seqs
    bt, ctx, tables, ctx_np = device_tables(bm, seqs)
    groups = bm.prefix_groups(seqs)
    assert len(groups[2]) == 8
    q = workloads.draw_queries(w, len(seqs), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = {}
    for kern in ("mma_sync", "tcgen05"):
        if kern == "tcgen05":
            monkeypatch.setenv("PAGEDKV_PREFIX_KERNEL", "tcgen05")
        else:
            monkeypatch.delenv("PAGEDKV_PREFIX_KERNEL", raising=False)
        outs[kern] = binding.decode_shared_prefix(q, k_pool, v_pool, bt, ctx, w.scale, groups,
                                                  dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle_decode_by_kv_head(q, k_pool, v_pool, tables, ctx_np, w.scale)
    for kern, out in outs.items():
        check_close(to_f64(out), want, w.dtype, f"{name}[{kern}]")
