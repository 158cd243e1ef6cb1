"""Pins for the reference block manager (CPU only).

* A hand-worked trace under ``tests/golden/block_manager_trace.txt`` (every
  expected value written out by hand from the rules on the pages).
* Invariants over seeded random operation sequences: counts equal table
  references, free + used = pool size, per-sequence tail waste below one block
  ("PagedAttention: Optimizing KV Cache in vLLM", section 2: waste is confined
  to the last block), failed calls change nothing ("What is PagedAttention?",
  How It Works).
* Copy-on-write isolation at the data level: a sibling's decode output is
  unchanged by another branch's copy + append (grasp.study section 4;
  qubittool, Share Without Mutating State).
"""

import os

import numpy as np
import pytest

import oracle
from oracle.block_manager import BlockManager, InvalidArgument, NoFreeBlocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "block_manager_trace.txt")


class TraceRunner:
    """Drives a block-manager implementation through the golden trace.

    ``make(nb, bs, mbs, order)`` builds a manager; the adapter methods below
    map trace ops onto it. Used for both the oracle and the C++ library.
    """

    def __init__(self, make):
        self.make = make
        self.bm = None

    def run(self, path=GOLDEN):
        checked = 0
        with open(path) as f:
            for raw in f:
                line = raw.split("#", 1)[0].strip()
                if not line:
                    continue
                checked += self.step(line)
        return checked

    def step(self, line):
        if line.startswith("init "):
            v = [int(x) for x in line.split()[1:]]
            self.bm = self.make(v[0], v[1], v[2], v[3:])
            return 0
        if line.startswith("expect"):
            return self.expect(line.split()[1:])
        lhs, rhs = [p.strip() for p in line.split("->")]
        op, *args = lhs.split()
        args = [int(a) for a in args]
        exp = rhs.split()
        if exp[0] == "nofree":
            with pytest.raises(NoFreeBlocks):
                self.call(op, args)
            return 1
        res = self.call(op, args)
        if exp[0] == "ok":
            return 1
        if exp[0] == "slot":
            slot, cs, cd = int(exp[1]), int(exp[3]), int(exp[4])
            assert (res.slot, res.cow_src, res.cow_dst) == (slot, cs, cd), line
            return 1
        if exp[0] == "slots":
            n = len(args)
            slots = [int(x) for x in exp[1:1 + n]]
            cows = [int(x) for x in exp[2 + n:2 + 3 * n]]
            assert [r.slot for r in res] == slots, line
            assert [c for r in res for c in (r.cow_src, r.cow_dst)] == cows, line
            return 1
        raise AssertionError(f"bad trace line {line}")

    def call(self, op, args):
        bm = self.bm
        if op == "allocate":
            return bm.allocate(args[0], args[1])
        if op == "fork":
            return bm.fork(args[0], args[1])
        if op == "append":
            return bm.append_slot(args[0])
        if op == "appends":
            return bm.append_slots(args)
        if op == "free":
            return bm.free(args[0])
        raise AssertionError(op)

    def expect(self, toks):
        what, vals = toks[0], [int(x) for x in toks[1:]]
        bm = self.bm
        if what == "table":
            assert list(bm.block_table(vals[0])) == vals[1:], toks
        elif what == "free":
            assert list(bm.free_queue_list()) == vals, toks
        elif what == "refcount":
            assert bm.refcount_of(vals[0]) == vals[1], toks
        elif what == "refcounts":
            assert [bm.refcount_of(b) for b in range(len(vals))] == vals, toks
        elif what == "context":
            assert bm.context_len(vals[0]) == vals[1], toks
        elif what == "cow_copies":
            assert bm.stats()["cow_copies"] == vals[0], toks
        else:
            raise AssertionError(f"bad expectation {toks}")
        return 1


class _OracleAdapter(BlockManager):
    def free_queue_list(self):
        return list(self.free_queue)

    def refcount_of(self, b):
        return self.refcount[b]


def test_golden_trace_oracle():
    runner = TraceRunner(lambda nb, bs, mbs, order: _OracleAdapter(nb, bs, mbs, order))
    assert runner.run() > 40


def _check_invariants(bm: BlockManager):
    counts = np.zeros(bm.num_blocks, dtype=np.int64)
    for table in bm.tables.values():
        for b in table:
            if b >= 0:
                counts[b] += 1
    assert list(counts) == list(bm.refcount)
    used = int(np.sum(counts > 0))
    assert used + len(bm.free_queue) == bm.num_blocks
    assert len(set(bm.free_queue)) == len(bm.free_queue)
    assert all(bm.refcount[b] == 0 for b in bm.free_queue)
    for s, table in bm.tables.items():
        ctx = bm.context[s]
        waste = len(table) * bm.block_size - ctx
        assert 0 <= waste <= bm.block_size - 1 or (ctx == 0 and len(table) == 0)
        assert len(table) <= bm.max_blocks_per_seq
        released = [i for i, b in enumerate(table) if b < 0]
        assert released == list(range(len(released)))   # only a leading run is released


def random_ops(seed, n_ops=400, num_blocks=40, block_size=4, mbs=12):
    """Seeded random op list (allocate / fork / append / appends / free)."""
    rng = np.random.default_rng(seed)
    ops = []
    next_id = 0
    live = []
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.2 or not live:
            ops.append(("allocate", next_id, int(rng.integers(0, 3 * block_size * 2))))
            live.append(next_id)
            next_id += 1
        elif r < 0.35:
            ops.append(("fork", int(rng.choice(live)), next_id))
            live.append(next_id)
            next_id += 1
        elif r < 0.7:
            ops.append(("append", int(rng.choice(live))))
        elif r < 0.8:
            k = int(rng.integers(1, min(4, len(live)) + 1))
            ops.append(("appends",) + tuple(int(x) for x in rng.choice(live, size=k, replace=False)))
        elif r < 0.85:
            # sliding window: release everything before a random token position
            ops.append(("release", int(rng.choice(live)), int(rng.integers(0, 4 * block_size * 2))))
        elif r < 0.9:
            # preemption by swap, and bringing a sequence back
            ops.append((("swap_out", "swap_in")[int(rng.integers(0, 2))], int(rng.choice(live))))
        else:
            victim = int(rng.choice(live))
            ops.append(("free", victim))
            live.remove(victim)
    order = rng.permutation(num_blocks).astype(np.int32)
    return (num_blocks, block_size, mbs, order), ops


def apply_op(bm, op):
    kind = op[0]
    try:
        if kind == "allocate":
            bm.allocate(op[1], op[2])
        elif kind == "fork":
            bm.fork(op[1], op[2])
        elif kind == "append":
            r = bm.append_slot(op[1])
            return ("ok", (r.slot, r.cow_src, r.cow_dst))
        elif kind == "appends":
            rs = bm.append_slots(list(op[1:]))
            return ("ok", tuple((r.slot, r.cow_src, r.cow_dst) for r in rs))
        elif kind == "free":
            bm.free(op[1])
        elif kind == "release":
            first = min(op[2], bm.context_len(op[1]))
            r = bm.release_before(op[1], first)
            return ("ok", len(r) if isinstance(r, list) else r)
        elif kind == "swap_out":
            return ("ok", tuple(bm.swap_out(op[1])))
        elif kind == "swap_in":
            return ("ok", tuple(bm.swap_in(op[1])))
        return ("ok", None)
    except NoFreeBlocks:
        return ("nofree", None)
    except InvalidArgument:
        return ("invalid", None)


@pytest.mark.parametrize("seed", range(6))
def test_invariants_and_atomic_failure(seed):
    (nb, bs, mbs, order), ops = random_ops(seed)
    bm = BlockManager(nb, bs, mbs, order)
    fails = 0
    for op in ops:
        before = bm.snapshot()
        status, _ = apply_op(bm, op)
        if status != "ok":
            fails += 1
            assert bm.snapshot() == before, op
        _check_invariants(bm)
    assert fails > 0  # the sequence exercises the failure path


def test_cow_isolation_of_sibling_outputs():
    rng = np.random.default_rng(11)
    nb, H, bs, D = 10, 2, 4, 8
    bm = BlockManager(nb, bs, 4, rng.permutation(nb))
    k_pool = rng.standard_normal((nb, H, bs, D))
    v_pool = rng.standard_normal((nb, H, bs, D))
    bm.allocate(0, 6)                 # tail block holds 2 tokens
    bm.fork(0, 1)
    bm.fork(0, 2)
    q = rng.standard_normal((3, H, D))

    def outputs(seqs):
        tables = np.array([bm.block_table(s) + [-1] * (4 - len(bm.block_table(s))) for s in seqs])
        lens = np.array([bm.context_len(s) for s in seqs])
        return oracle.paged_decode(q[:len(seqs)], k_pool, v_pool, tables, lens, 0.3)

    before = outputs([1, 2])
    res = bm.append_slot(0)
    assert res.cow_src >= 0 and res.cow_dst >= 0
    oracle.copy_blocks(k_pool, v_pool, [(res.cow_src, res.cow_dst)])
    oracle.kv_append(k_pool, v_pool, rng.standard_normal((1, H, D)),
                     rng.standard_normal((1, H, D)), [res.slot])
    after = outputs([1, 2])
    assert np.array_equal(before, after)
    # the writer's copy holds the shared tokens plus its new one
    t0 = bm.block_table(0)
    assert np.array_equal(k_pool[t0[-1], :, :2], k_pool[res.cow_src, :, :2])


def test_waste_bound_over_growth():
    bm = BlockManager(64, 16, 64)
    bm.allocate(0, 1)
    for _ in range(500):
        bm.append_slot(0)
        waste = len(bm.block_table(0)) * 16 - bm.context_len(0)
        assert 0 <= waste <= 15


def test_rejects_bad_arguments():
    bm = BlockManager(4, 4, 2)
    with pytest.raises(InvalidArgument):
        bm.allocate(0, 9)              # 3 blocks > max_blocks_per_seq
    bm.allocate(0, 8)
    with pytest.raises(InvalidArgument):
        bm.append_slot(0)              # full tail and table at capacity
    with pytest.raises(InvalidArgument):
        bm.allocate(0, 1)              # duplicate id
    with pytest.raises(InvalidArgument):
        bm.fork(7, 8)                  # unknown parent
    with pytest.raises(InvalidArgument):
        BlockManager(3, 4, 2, [0, 0, 1])


def test_release_before_hand_example():
    bm = BlockManager(8, 4, 6, [3, 1, 4, 0, 5, 2, 6, 7])
    bm.allocate(0, 10)             # blocks 3, 1, 4
    bm.fork(0, 1)                  # shared: counts 2
    assert bm.release_before(0, 9) == []          # blocks 0,1 of seq 0 out: 3, 1 still held by seq 1
    assert bm.block_table(0) == [-1, -1, 4]
    assert bm.refcount[3] == 1 and bm.refcount[1] == 1
    assert bm.release_before(1, 4) == [3]         # seq 1 drops block 3 (count 0 -> reclaimed)
    assert bm.block_table(1) == [-1, 1, 4]
    assert list(bm.free_queue) == [0, 5, 2, 6, 7, 3]
    st = bm.stats()
    assert st["logical_slots"] == 3 * 4 and st["logical_tokens"] == (10 - 8) + (10 - 4)
    bm.free(0)
    bm.free(1)
    assert sorted(bm.free_queue) == list(range(8))


def test_swap_hand_example():
    bm = BlockManager(6, 4, 4, [2, 5, 0, 1, 3, 4])
    bm.allocate(0, 6)              # blocks 2, 5
    bm.fork(0, 1)                  # shared
    assert bm.swap_out(0) == [2, 5]          # still held by seq 1: nothing reclaimed
    assert bm.block_table(0) == [-1, -1] and bm.context_len(0) == 6
    assert list(bm.free_queue) == [0, 1, 3, 4]
    with pytest.raises(InvalidArgument):
        bm.append_slot(0)                    # swapped out
    bm.allocate(2, 12)                       # takes 0, 1, 3
    with pytest.raises(NoFreeBlocks):
        bm.swap_in(0)                        # needs 2, one free: nothing changes
    assert bm.block_table(0) == [-1, -1]
    bm.free(1)                               # reclaims 2, 5
    assert bm.swap_in(0) == [4, 2]           # private copies, in queue order
    assert bm.refcount[4] == 1 and bm.refcount[2] == 1
    assert bm.append_slot(0).slot == 2 * 4 + 2   # appends go on as before
