"""GPU parity of every kernel against the CPU oracle, through the C ABI.

Small ragged cases spanning several blocks, partitions and a ragged tail are
compared element by element; invariants the pages fix are checked on the GPU
path itself (placement independence, copy-on-write isolation, single token,
identical keys). Tolerances: fp32 max-abs 1e-5; bf16 max-abs 2e-2 and
mean-abs 2e-3 against the float64 oracle. Append and copy are bit-exact.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads
from paged_kv_cache_336_b200.binding import BlockManager

from gpu_util import (build_tables, check_close, device_tables, setup, to_f64)

pytestmark = pytest.mark.gpu


def _err_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _run_decode(kind, q, k_pool, v_pool, bt, ctx, scale, partition=512, err=None):
    """kind: "decode" (pa_decode), "split" (pa_decode_split, the kernel the
    library picks), "split_ticket" / "split_stream" (pa_decode_split on the
    partition-ticket or the balanced kernel)."""
    if kind == "decode":
        return binding.decode(q, k_pool, v_pool, bt, ctx, scale, dev_err=err)
    prev = os.environ.get("PAGEDKV_SPLIT_KERNEL")
    if kind != "split":
        os.environ["PAGEDKV_SPLIT_KERNEL"] = kind.split("_")[1]
    try:
        return binding.decode_split(q, k_pool, v_pool, bt, ctx, scale, partition_tokens=partition,
                                    dev_err=err)
    finally:
        if prev is None:
            os.environ.pop("PAGEDKV_SPLIT_KERNEL", None)
        else:
            os.environ["PAGEDKV_SPLIT_KERNEL"] = prev


def _full_oracle(q, k_pool, v_pool, tables, ctx, scale):
    return oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx, scale)


CASES = [
    # dtype, Hq, Hkv, D, bs
    (workloads.F32, 2, 2, 64, 16),
    (workloads.F32, 4, 2, 128, 16),
    (workloads.F32, 8, 1, 64, 32),
    (workloads.F32, 16, 2, 128, 32),
    (workloads.BF16, 4, 4, 128, 16),
    (workloads.BF16, 2, 2, 64, 32),
    (workloads.BF16, 2, 2, 256, 16),
    (workloads.BF16, 16, 2, 128, 16),
    (workloads.BF16, 8, 2, 64, 16),
    (workloads.BF16, 12, 4, 128, 32),
    (workloads.BF16, 32, 2, 128, 16),
    (workloads.BF16, 6, 3, 256, 32),
]


@pytest.mark.parametrize("kind", ["decode", "split_ticket", "split_stream"])
@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", CASES)
def test_decode_matches_oracle_small(kind, dtype, Hq, Hkv, D, bs):
    w = workloads.random_small(1000 + Hq * 7 + D + bs, num_seqs=7, num_q_heads=Hq,
                               num_kv_heads=Hkv, head_dim=D, block_size=bs, dtype=dtype,
                               max_ctx=9 * bs + 5,
                               fixed_lens=[0, 1, bs, 9 * bs + 5])  # empty, 1 token, 1 block, longest
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 7, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(7)))
    err = _err_word()
    out = _run_decode(kind, q, k_pool, v_pool, bt, ctx, w.scale, partition=2 * bs, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale)
    check_close(to_f64(out), want, dtype, f"{kind} {dtype} Hq={Hq} Hkv={Hkv} D={D} bs={bs}")
    assert torch.all(out[0] == 0)  # empty context gives zeros


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("G", [1, 8])
def test_long_table_shape_matches_oracle(bs, G):
    """Tables sized for >= 32k tokens select the deep CTA shape (2 warps x 3
    stages); small contexts keep the comparison cheap."""
    w = workloads.random_small(88 + G + bs, num_seqs=6, num_q_heads=2 * G, num_kv_heads=2,
                               head_dim=128, block_size=bs, dtype=workloads.BF16,
                               max_ctx=40 * bs, fixed_lens=[0, 1, 40 * bs, 17])
    w.max_blocks_per_seq = 32768 // bs + 3
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 6, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(6)))
    want = _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale)
    for kind in ("decode", "split_ticket", "split_stream"):
        out = _run_decode(kind, q, k_pool, v_pool, bt, ctx, w.scale, partition=3 * bs)
        check_close(to_f64(out), want, w.dtype, f"deep {kind}")


@pytest.mark.parametrize("dtype,G", [(workloads.F32, 1), (workloads.BF16, 1), (workloads.BF16, 8)])
@pytest.mark.parametrize("partition_blocks", [1, 2, 3, 5, 64])
@pytest.mark.parametrize("kind", ["split_ticket", "split_stream"])
def test_split_any_partition_equals_oracle(kind, dtype, G, partition_blocks):
    bs = 16
    w = workloads.random_small(77 + partition_blocks, num_seqs=5, num_q_heads=2 * G,
                               num_kv_heads=2, head_dim=128, block_size=bs, dtype=dtype,
                               max_ctx=20 * bs,
                               fixed_lens=[5 * bs, 5 * bs + 1, 20 * bs])  # exact and ragged edges
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 5, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(5)))
    out = _run_decode(kind, q, k_pool, v_pool, bt, ctx, w.scale, partition=partition_blocks * bs)
    ref = binding.decode(q, k_pool, v_pool, bt, ctx, w.scale)
    want = _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale)
    check_close(to_f64(out), want, dtype, kind)
    check_close(to_f64(ref), want, dtype, "unsplit")


def test_tiny_workload_full_step():
    """The tiny fp32 workload: prefill, fork(3->4), one appended token per
    sequence 0..3 (sequence 3 copies its shared tail), decode 0..4."""
    w = workloads.tiny()
    bm, k_pool, v_pool = setup(w)
    ref_bm = oracle.BlockManager(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
    build_tables(ref_bm, w)
    k_ref, v_ref = to_f64(k_pool), to_f64(v_pool)
    # host step
    slots, pairs = bm.append_slots_arrays(w.step_seqs)
    r = ref_bm.append_slots(w.step_seqs)
    assert slots.tolist() == [x.slot for x in r]
    assert pairs.tolist() == [[x.cow_src, x.cow_dst] for x in r if x.cow_src >= 0]
    assert len(pairs) == 1
    k_new, v_new = workloads.draw_new_kv(w, len(w.step_seqs), device="cuda")
    err = _err_word()
    binding.copy_blocks(k_pool, v_pool, torch.from_numpy(pairs).cuda(), dev_err=err)
    binding.kv_append(k_new, v_new, torch.from_numpy(slots).cuda(), k_pool, v_pool, dev_err=err)
    oracle.copy_blocks(k_ref, v_ref, pairs)
    oracle.kv_append(k_ref, v_ref, to_f64(k_new), to_f64(v_new), slots)
    assert np.array_equal(to_f64(k_pool), k_ref) and np.array_equal(to_f64(v_pool), v_ref)
    bt, ctx, tables, ctx_np = device_tables(bm, w.decode_seqs)
    assert ctx_np.tolist() == [2, 16, 17, 34, 33]
    q = workloads.draw_queries(w, len(w.decode_seqs), device="cuda")
    want = _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale)
    for kind in ("decode", "split_ticket", "split_stream"):
        out = _run_decode(kind, q, k_pool, v_pool, bt, ctx, w.scale, partition=16, err=err)
        check_close(to_f64(out), want, w.dtype, kind)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


@pytest.mark.parametrize("dtype", [workloads.F32, workloads.BF16])
def test_kv_append_bit_exact(dtype):
    torch.manual_seed(0)
    tdt = torch.float32 if dtype == workloads.F32 else torch.bfloat16
    NB, H, bs, D = 9, 4, 16, 128
    k_pool = torch.randn(NB, H, bs, D, device="cuda").to(tdt)
    v_pool = torch.randn(NB, H, bs, D, device="cuda").to(tdt)
    T = 6
    k_new = torch.randn(T, H, D, device="cuda").to(tdt)
    v_new = torch.randn(T, H, D, device="cuda").to(tdt)
    slots = torch.tensor([0, 37, -1, 143, 15, 80], dtype=torch.int64, device="cuda")
    idt = torch.int16 if tdt == torch.bfloat16 else torch.int32   # compare bit patterns
    kr, vr = k_pool.view(idt).cpu().numpy(), v_pool.view(idt).cpu().numpy()
    kn, vn = k_new.view(idt).cpu().numpy(), v_new.view(idt).cpu().numpy()
    oracle.kv_append(kr, vr, kn, vn, slots.cpu().numpy())
    err = _err_word()
    binding.kv_append(k_new, v_new, slots, k_pool, v_pool, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(k_pool.view(idt).cpu().numpy(), kr)
    assert np.array_equal(v_pool.view(idt).cpu().numpy(), vr)


@pytest.mark.parametrize("dtype", [workloads.F32, workloads.BF16])
def test_copy_blocks_bit_exact(dtype):
    torch.manual_seed(1)
    tdt = torch.float32 if dtype == workloads.F32 else torch.bfloat16
    NB, H, bs, D = 12, 8, 16, 128
    k_pool = torch.randn(NB, H, bs, D, device="cuda").to(tdt)
    v_pool = torch.randn(NB, H, bs, D, device="cuda").to(tdt)
    pairs = np.array([[3, 7], [0, 11], [5, 2]], dtype=np.int64)
    idt = torch.int16 if tdt == torch.bfloat16 else torch.int32   # compare bit patterns
    k_ref, v_ref = k_pool.view(idt).cpu().numpy(), v_pool.view(idt).cpu().numpy()
    oracle.copy_blocks(k_ref, v_ref, pairs)
    err = _err_word()
    binding.copy_blocks(k_pool, v_pool, torch.from_numpy(pairs).cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(k_pool.view(idt).cpu().numpy(), k_ref)
    assert np.array_equal(v_pool.view(idt).cpu().numpy(), v_ref)


def test_device_error_word_and_skipped_accesses():
    w = workloads.random_small(5, num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=60, min_ctx=40)
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 3, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, [0, 1, 2])
    # a block id past the pool in sequence 1
    bt_bad = bt.clone()
    bt_bad[1, 1] = w.num_blocks + 5
    for kind in ("decode", "split_ticket", "split_stream"):
        err = _err_word()
        out = _run_decode(kind, q, k_pool, v_pool, bt_bad, ctx, w.scale, partition=32, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) & binding.DEVERR_BLOCK_ID
        assert torch.isfinite(out.float()).all()
        want = oracle.paged_decode(to_f64(q), to_f64(k_pool), to_f64(v_pool), tables, ctx_np,
                                   w.scale)
        check_close(to_f64(out[[0, 2]]), want[[0, 2]], w.dtype, "untouched rows")
    # a context length past max_blocks_per_seq * block_size
    ctx_bad = ctx.clone()
    ctx_bad[2] = w.max_blocks_per_seq * w.block_size + 1
    err = _err_word()
    out = binding.decode(q, k_pool, v_pool, bt, ctx_bad, w.scale, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & binding.DEVERR_CONTEXT_LEN
    assert torch.all(out[2] == 0)
    # a slot past the pool, and a copy pair past the pool
    err = _err_word()
    k_before = k_pool.clone()
    slots = torch.tensor([w.num_blocks * w.block_size + 3], dtype=torch.int64, device="cuda")
    kn = torch.ones(1, 2, 128, dtype=k_pool.dtype, device="cuda")
    binding.kv_append(kn, kn, slots, k_pool, v_pool, dev_err=err)
    binding.copy_blocks(k_pool, v_pool, torch.tensor([[0, w.num_blocks]], device="cuda"), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & binding.DEVERR_SLOT
    assert int(err.item()) & binding.DEVERR_COPY_PAIR
    assert torch.equal(k_pool, k_before)


@pytest.mark.parametrize("dtype,G", [(workloads.F32, 1), (workloads.BF16, 1), (workloads.BF16, 8)])
def test_gpu_output_independent_of_physical_placement(dtype, G):
    w = workloads.random_small(9, num_seqs=4, num_q_heads=2 * G, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=dtype, max_ctx=200, min_ctx=20)
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 4, device="cuda")
    bt, ctx, tables, _ = device_tables(bm, [0, 1, 2, 3])
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(3)).cuda()
    k2 = torch.empty_like(k_pool)
    v2 = torch.empty_like(v_pool)
    k2[perm] = k_pool
    v2[perm] = v_pool
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].int(), bt)
    for kind in ("decode", "split_ticket", "split_stream"):
        a = _run_decode(kind, q, k_pool, v_pool, bt, ctx, w.scale, partition=48)
        b = _run_decode(kind, q, k2, v2, bt2, ctx, w.scale, partition=48)
        assert torch.equal(a, b), kind


@pytest.mark.parametrize("dtype,G", [(workloads.F32, 1), (workloads.BF16, 1), (workloads.BF16, 4)])
def test_single_token_returns_v_exactly(dtype, G):
    w = workloads.random_small(11, num_seqs=3, num_q_heads=2 * G, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=dtype, max_ctx=1, min_ctx=1)
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 3, device="cuda") * 30
    bt, ctx, tables, _ = device_tables(bm, [0, 1, 2])
    for kind in ("decode", "split_ticket", "split_stream"):
        out = _run_decode(kind, q, k_pool, v_pool, bt, ctx, w.scale, partition=16)
        for s in range(3):
            b = int(tables[s, 0])
            want = v_pool[b, :, 0, :].repeat_interleave(G, dim=0)
            assert torch.equal(out[s], want), (kind, s)


def test_identical_keys_give_mean_of_values():
    w = workloads.random_small(12, num_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.F32, max_ctx=300, min_ctx=100)
    bm, k_pool, v_pool = setup(w)
    k_pool[:] = k_pool[0, :, 0:1, :]   # one key everywhere (per head)
    q = workloads.draw_queries(w, 2, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, [0, 1])
    out = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=64)
    vp = to_f64(v_pool)
    for s in range(2):
        nb = -(-int(ctx_np[s]) // 16)
        vals = vp[tables[s, :nb]].transpose(1, 0, 2, 3).reshape(2, nb * 16, 128)[:, :ctx_np[s]]
        mean = vals.mean(axis=1).repeat(4, axis=0)
        check_close(to_f64(out[s]), mean, workloads.F32, "mean of V")


def test_large_logits_stay_finite():
    w = workloads.random_small(13, num_seqs=3, num_q_heads=8, num_kv_heads=1, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=500, min_ctx=100)
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 3, device="cuda") * 40.0   # logits of order 1e2..1e3
    bt, ctx, tables, ctx_np = device_tables(bm, [0, 1, 2])
    out = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=128)
    assert torch.isfinite(out.float()).all()
    want = _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale)
    check_close(to_f64(out), want, w.dtype, "large logits")


def test_cow_isolation_on_gpu():
    """A branch's copy-on-write and append leave its siblings' outputs
    unchanged: bit for bit on pa_decode (one CTA per sequence and KV head, so
    a sequence's arithmetic does not depend on the rest of the batch), and
    within the tolerance on pa_decode_split, whose even cut of the batch's
    work moves piece boundaries when another sequence grows (both against
    the oracle too)."""
    w = workloads.random_small(14, num_seqs=1, num_q_heads=16, num_kv_heads=4, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=0, spare_blocks=12)
    bm = BlockManager(w.num_blocks, 16, 8, w.free_order)
    k_pool, v_pool = workloads.draw_pools(w, "cuda")
    bm.allocate(0, 41)                 # tail block holds 9 tokens
    for c in (1, 2, 3):
        bm.fork(0, c)
    q = workloads.draw_queries(w, 4, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, [0, 1, 2, 3])
    before = {kind: _run_decode(kind, q, k_pool, v_pool, bt, ctx, w.scale, partition=32)
              for kind in ("decode", "split_ticket", "split_stream")}
    want_before = _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale)
    slots, pairs = bm.append_slots_arrays([2])
    assert len(pairs) == 1
    binding.copy_blocks(k_pool, v_pool, torch.from_numpy(pairs).cuda())
    kn, vn = workloads.draw_new_kv(w, 1, device="cuda")
    binding.kv_append(kn, vn, torch.from_numpy(slots).cuda(), k_pool, v_pool)
    bt2, ctx2, tables2, ctx2_np = device_tables(bm, [0, 1, 2, 3])
    want_after = _full_oracle(q, k_pool, v_pool, tables2, ctx2_np, w.scale)
    for s in (0, 1, 3):   # the oracle's siblings are unchanged, bit for bit
        assert np.array_equal(want_before[s], want_after[s]), s
    for kind in ("decode", "split_ticket", "split_stream"):
        after = _run_decode(kind, q, k_pool, v_pool, bt2, ctx2, w.scale, partition=32)
        check_close(to_f64(after), want_after, w.dtype, f"after the copy [{kind}]")
        for s in (0, 1, 3):
            if kind == "decode":
                assert torch.equal(before[kind][s], after[s]), (kind, s)
            check_close(to_f64(after[s]), to_f64(before[kind][s]), w.dtype, f"sibling {s} [{kind}]")
        assert not torch.equal(before[kind][2], after[2])


def test_repeated_split_calls_reuse_workspace():
    """The workspace header (the ticket kernel's counters) is zero again after
    every call, and repeated calls give the same result."""
    w = workloads.random_small(15, num_seqs=9, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=workloads.BF16, max_ctx=700)
    bm, k_pool, v_pool = setup(w)
    q = workloads.draw_queries(w, 9, device="cuda")
    bt, ctx, tables, ctx_np = device_tables(bm, list(range(9)))
    ws = binding.SplitWorkspace(9, 8, 128, 16, w.max_blocks_per_seq, 64)
    outs = [binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=64,
                                 workspace=ws) for _ in range(5)]
    torch.cuda.synchronize()
    header = ws.buffer[ws.ptr - ws.buffer.data_ptr():][:8]   # the two uint32 counters
    assert int(header.sum().item()) == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    want = _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale)
    check_close(to_f64(outs[0]), want, w.dtype, "reused workspace")


def test_host_validation_flag_rejects_bad_tables():
    """PAGEDKV_VALIDATE=1 copies the tables and lengths to the host and rejects
    an out-of-range entry before launching, and refuses copy lists with a
    repeated destination or a block that is both source and destination (the
    flag is read once per process, so the check runs in a child)."""
    import subprocess
    import sys
    import textwrap
    code = textwrap.dedent("""
        import sys, torch
        sys.path.insert(0, %r)
        sys.path.insert(0, %r)
        from paged_kv_cache_336_b200 import binding, workloads
        from gpu_util import setup, device_tables
        w = workloads.random_small(3, num_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=128,
                                   block_size=16, dtype=workloads.BF16, max_ctx=60, min_ctx=20)
        bm, k, v = setup(w)
        q = workloads.draw_queries(w, 3, device="cuda")
        bt, ctx, _, _ = device_tables(bm, [0, 1, 2])
        binding.decode(q, k, v, bt, ctx, w.scale)          # valid tables pass
        bt[1, 0] = w.num_blocks + 3
        try:
            binding.decode_split(q, k, v, bt, ctx, w.scale, partition_tokens=32)
        except binding.InvalidArgumentError as e:
            assert "block_tables[1][0]" in str(e), e
            print("rejected")
        # copy lists whose result would depend on the order of the copies
        assert w.num_blocks > 6
        binding.copy_blocks(k, v, torch.tensor([[0, 5], [1, 6]], device="cuda"))   # fine
        for pairs, why in (([[0, 5], [1, 5]], "twice"), ([[0, 5], [5, 6]], "both a source")):
            try:
                binding.copy_blocks(k, v, torch.tensor(pairs, device="cuda"))
            except binding.InvalidArgumentError as e:
                assert why in str(e), e
                print("pairs rejected")
    """) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
            os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PAGEDKV_VALIDATE="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "rejected" in r.stdout
    assert r.stdout.count("pairs rejected") == 2


@pytest.mark.parametrize("Hq,Hkv,dtype", [(6, 3, workloads.BF16), (32, 32, workloads.BF16),
                                          (16, 16, workloads.F32), (40, 5, workloads.BF16)])
def test_balanced_split_kv_head_counts(Hq, Hkv, dtype):
    """The balanced kernel's warp groups are Hkv warps wide: KV-head counts
    that do not divide a CTA's warps (3, 5), and ones larger than a CTA (16,
    32), against the oracle (the kernel forced for these short tables)."""
    os.environ["PAGEDKV_SPLIT_KERNEL"] = "stream"
    try:
        w = workloads.random_small(120 + Hkv, num_seqs=5, num_q_heads=Hq, num_kv_heads=Hkv,
                                   head_dim=128, block_size=16, dtype=dtype, max_ctx=900,
                                   fixed_lens=[0, 1, 900])
        bm, k_pool, v_pool = setup(w)
        q = workloads.draw_queries(w, 5, device="cuda")
        bt, ctx, tables, ctx_np = device_tables(bm, list(range(5)))
        err = _err_word()
        out = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=64,
                                   dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        check_close(to_f64(out), _full_oracle(q, k_pool, v_pool, tables, ctx_np, w.scale), dtype,
                    f"Hq={Hq} Hkv={Hkv}")
    finally:
        os.environ.pop("PAGEDKV_SPLIT_KERNEL", None)


def test_balanced_split_many_sequences():
    """4096 sequences (the most pa_decode_split takes) of 0..40 tokens in
    tables that hold 32768 tokens: the per-sequence arrays fill the balanced
    kernel's shared memory; every output against the oracle."""
    B, bs, mbs = 4096, 16, 2048
    rng = np.random.default_rng(77)
    ctx_np = rng.integers(0, 41, size=B).astype(np.int32)
    nb = int(np.sum((ctx_np + bs - 1) // bs)) + 8
    order = rng.permutation(nb).astype(np.int32)
    bm = BlockManager(nb, bs, mbs, order)
    for s in range(B):
        bm.allocate(s, int(ctx_np[s]))
    w = workloads.random_small(78, num_seqs=1, num_q_heads=4, num_kv_heads=2, head_dim=128,
                               block_size=bs, dtype=workloads.BF16, max_ctx=1)
    w.num_blocks = nb
    k_pool, v_pool = workloads.draw_pools(w, "cuda")
    q = workloads.draw_queries(w, B, device="cuda")
    bt, ctx, tables, ctx2 = device_tables(bm, list(range(B)))
    err = _err_word()
    out = binding.decode_split(q, k_pool, v_pool, bt, ctx, w.scale, partition_tokens=512,
                               dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_close(to_f64(out), _full_oracle(q, k_pool, v_pool, tables, ctx2, w.scale), w.dtype,
                "4096 sequences")
    assert torch.all(out[torch.from_numpy(ctx2 == 0).cuda()] == 0)
