"""pa_decode_step (one whole decode step from host buffers) against the oracle
over several consecutive steps with copy-on-write: outputs within the decode
tolerances, pools bit-exact, copy counts equal to the reference manager's."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_336_b200 import binding, workloads

from gpu_util import check_close, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,Hq,Hkv,bs", [(workloads.BF16, 8, 2, 16), (workloads.F32, 2, 2, 32),
                                              (workloads.BF16, 4, 4, 32)])
def test_decode_step_matches_oracle(dtype, Hq, Hkv, bs):
    D, NB, MBS = 128, 40, 8
    rng = np.random.default_rng(21)
    order = rng.permutation(NB).astype(np.int32)
    lib_bm = binding.BlockManager(NB, bs, MBS, order)
    ref_bm = oracle.BlockManager(NB, bs, MBS, order)
    for m in (lib_bm, ref_bm):
        m.allocate(0, 2 * bs + 5)      # partial tail, shared by 1 and 2 below
        m.allocate(3, 3 * bs)          # full tail: next append takes a new block
        m.allocate(4, 1)
        m.fork(0, 1)
        m.fork(0, 2)
    w = workloads.random_small(5, num_seqs=1, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=dtype, max_ctx=1)
    w.num_blocks = NB
    k_pool, v_pool = workloads.draw_pools(w, "cuda")
    k_ref, v_ref = to_f64(k_pool), to_f64(v_pool)
    scale = 1.0 / np.sqrt(D)
    stepper = binding.DecodeStepper(lib_bm, k_pool, v_pool, Hq, scale, max_seqs=8,
                                    partition_tokens=bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    seqs = np.array([2, 0, 3, 4, 1], dtype=np.int64)
    total_cow = 0
    for step in range(4):
        q = workloads.draw_queries(w, len(seqs), step=step).pin_memory()
        kn, vn = workloads.draw_new_kv(w, len(seqs), step=step)
        kn, vn = kn.pin_memory(), vn.pin_memory()
        out = torch.empty_like(q).pin_memory()
        ncow = stepper.step(seqs, q, kn, vn, out, dev_err=err)
        res = ref_bm.append_slots(seqs.tolist())
        pairs = [(r.cow_src, r.cow_dst) for r in res if r.cow_src >= 0]
        assert ncow == len(pairs)
        total_cow += ncow
        oracle.copy_blocks(k_ref, v_ref, pairs)
        oracle.kv_append(k_ref, v_ref, to_f64(kn), to_f64(vn), [r.slot for r in res])
        tables = np.full((len(seqs), MBS), -1, dtype=np.int64)
        for i, s in enumerate(seqs):
            t = ref_bm.block_table(int(s))
            tables[i, :len(t)] = t
        ctx = np.array([ref_bm.context_len(int(s)) for s in seqs])
        want = oracle.paged_decode(to_f64(q), k_ref, v_ref, tables, ctx, scale)
        check_close(to_f64(out), want, dtype, f"step {step}")
        assert stepper.h2d_bytes(len(seqs), ncow) > 0 and stepper.d2h_bytes(len(seqs)) == out.numel() * out.element_size()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert total_cow == 2          # sequences 2 and 0 copy; 1 is the last holder
    assert np.array_equal(to_f64(k_pool), k_ref) and np.array_equal(to_f64(v_pool), v_ref)


def _step_setup(seed, NB=60, bs=16, MBS=12, Hq=8, Hkv=2, D=128):
    order = np.random.default_rng(seed).permutation(NB).astype(np.int32)
    bm = binding.BlockManager(NB, bs, MBS, order)
    bm.allocate(0, 2 * bs + 5)
    bm.allocate(3, 3 * bs)
    bm.allocate(4, 1)
    bm.fork(0, 1)
    bm.fork(0, 2)
    w = workloads.random_small(seed, num_seqs=1, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=workloads.BF16, max_ctx=1)
    w.num_blocks = NB
    k_pool, v_pool = workloads.draw_pools(w, "cuda")
    return bm, w, k_pool, v_pool


def test_pipelined_steps_equal_synchronous_steps():
    """Two buffer sets alternated with synchronize = 0, uploads on a copy
    stream (pa_step_pipeline_create): every step's output, the copy counts
    and the final pools are bit-identical to one-at-a-time synchronous steps
    from the same start."""
    Hq, D, steps = 8, 128, 10
    seqs = np.array([2, 0, 3, 4, 1], dtype=np.int64)
    scale = 1.0 / np.sqrt(D)
    runs = []
    for piped in (False, True):
        bm, w, k_pool, v_pool = _step_setup(33)
        inputs = []
        for step in range(steps):
            q = workloads.draw_queries(w, len(seqs), step=step).pin_memory()
            kn, vn = workloads.draw_new_kv(w, len(seqs), step=step)
            inputs.append((q, kn.pin_memory(), vn.pin_memory()))
        outs = [torch.empty_like(inputs[0][0]).pin_memory() for _ in range(steps)]
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if piped:
            copy_stream = torch.cuda.Stream()
            sets = [binding.DecodeStepper(bm, k_pool, v_pool, Hq, scale, max_seqs=8,
                                          partition_tokens=16, copy_stream=copy_stream)
                    for _ in range(2)]
        else:
            sets = [binding.DecodeStepper(bm, k_pool, v_pool, Hq, scale, max_seqs=8,
                                          partition_tokens=16)]
        stream = torch.cuda.current_stream()
        cows = []
        for step in range(steps):
            q, kn, vn = inputs[step]
            cows.append(sets[step % len(sets)].step(seqs, q, kn, vn, outs[step],
                                                    synchronize=not piped, dev_err=err,
                                                    stream=stream))
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        runs.append((cows, [o.clone() for o in outs], k_pool.clone().cpu(), v_pool.clone().cpu()))
    (c0, o0, k0, v0), (c1, o1, k1, v1) = runs
    assert c0 == c1 and sum(c0) > 0
    for step in range(steps):
        assert torch.equal(o0[step], o1[step]), f"step {step}"
    assert torch.equal(k0, k1) and torch.equal(v0, v1)
