"""CPU tests of the C ABI (no GPU needed).

* The shared library loads and exports every function declared in
  include/pagedkv.h.
* The C++ block manager matches the Python reference manager bit for bit:
  the hand-worked golden trace, seeded random operation sequences (slots,
  copy pairs, tables, counts, free-queue order, statistics, failures), and
  the block tables of every synthetic workload.
* Kernel entry points reject bad arguments before touching the device.
"""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from oracle.block_manager import BlockManager as RefBM, InvalidArgument, NoFreeBlocks
from paged_kv_cache_336_b200 import binding, workloads
from paged_kv_cache_336_b200.binding import (
    BlockManager as LibBM, InvalidArgumentError, NoFreeBlocksError, PagedKVError)

from test_oracle_block_manager import TraceRunner, random_ops, apply_op, _check_invariants

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_\w+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = binding.library()
    names = declared_functions()
    assert len(names) >= 20
    for name in names:
        assert hasattr(lib, name), name
        assert name in binding._SIGNATURES, f"{name} has no binding signature"
    assert lib.pa_version().decode().startswith("pagedkv")
    assert lib.pa_status_string(2).decode() == "PA_ERR_NO_FREE_BLOCKS"


def test_library_is_built_for_sm100a_only():
    # the fatbin inside the library is produced by `-gencode arch=compute_100a,code=sm_100a`;
    # the build script is the single place that sets it
    from paged_kv_cache_336_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


class _LibAdapter:
    """Maps the library manager onto the oracle's exception types for the trace."""

    def __init__(self, *args):
        self.bm = LibBM(*args)

    def __getattr__(self, name):
        fn = getattr(self.bm, name)

        def call(*a, **k):
            try:
                return fn(*a, **k)
            except NoFreeBlocksError as e:
                raise NoFreeBlocks(str(e))
            except InvalidArgumentError as e:
                raise InvalidArgument(str(e))
        return call


def test_golden_trace_library():
    runner = TraceRunner(lambda nb, bs, mbs, order: _LibAdapter(nb, bs, mbs, order))
    assert runner.run() > 40


def _lib_state(bm: LibBM, seqs):
    tables = tuple(sorted((s, tuple(bm.block_table(s))) for s in seqs))
    ctx = tuple(sorted((s, bm.context_len(s)) for s in seqs))
    rc = tuple(bm.refcount_of(b) for b in range(bm.num_blocks))
    return (tuple(bm.free_queue_list()), rc, tables, ctx, bm.stats()["cow_copies"])


@pytest.mark.parametrize("seed", range(8))
def test_random_ops_match_reference(seed):
    (nb, bs, mbs, order), ops = random_ops(seed, n_ops=300)
    ref = RefBM(nb, bs, mbs, order)
    lib = _LibAdapter(nb, bs, mbs, order)
    for op in ops:
        r_ref = apply_op(ref, op)
        r_lib = apply_op(lib, op)
        assert r_ref == r_lib, op
        assert _lib_state(lib.bm, list(ref.tables)) == ref.snapshot(), op
        st = lib.bm.stats()
        want = ref.stats()
        for k, v in want.items():
            assert st[k] == v, (k, op)
    _check_invariants(ref)


def test_can_append_agrees_with_append():
    bm = LibBM(6, 4, 3, list(range(6)))
    bm.allocate(10, 5)
    bm.fork(10, 11)
    bm.fork(10, 12)
    bm.allocate(13, 12)
    assert not bm.can_append([10, 11, 12])
    with pytest.raises(NoFreeBlocksError):
        bm.append_slots([10, 11, 12])
    assert bm.can_append([12])
    bm.free(13)
    assert bm.can_append([10, 11, 12])
    slots, pairs = bm.append_slots_arrays([10, 11, 12])
    assert slots.tolist() == [21, 9, 5]
    assert pairs.tolist() == [[1, 5], [1, 2]]


def build_tables(bm, w):
    """Applies a workload's prefill/fork/extra-token plan to a manager."""
    for s in w.prefill_seqs:
        bm.allocate(s, int(w.context_lens[s]))
    for parent, child in w.forks:
        bm.fork(parent, child)
    for s, n in sorted(w.extra_tokens.items()):
        for _ in range(n):
            bm.append_slot(s)


@pytest.mark.parametrize("name", ["tiny", "mha", "gqa", "prefix", "prefix_cow"])
def test_workload_tables_match_reference(name):
    w = workloads.WORKLOADS[name]()
    ref = RefBM(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
    lib = LibBM(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
    build_tables(ref, w)
    build_tables(lib, w)
    seqs = sorted(ref.tables)
    tables, ctx = lib.export(seqs)
    for i, s in enumerate(seqs):
        t = ref.block_table(s)
        assert tables[i, :len(t)].tolist() == t
        assert (tables[i, len(t):] == -1).all()
        assert ctx[i] == ref.context_len(s)
    if w.step_seqs:
        r1 = ref.append_slots(w.step_seqs)
        slots, pairs = lib.append_slots_arrays(w.step_seqs)
        assert slots.tolist() == [r.slot for r in r1]
        want_pairs = [[r.cow_src, r.cow_dst] for r in r1 if r.cow_src >= 0]
        assert pairs.tolist() == want_pairs
        if name == "prefix_cow":
            assert len(want_pairs) == 8 * 15   # every branch but the last copies
        if name == "tiny":
            assert len(want_pairs) == 1        # sequence 3's shared tail is copied


def test_long_workload_tables_match_reference():
    w = workloads.long(block_size=32)
    ref = RefBM(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
    lib = LibBM(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
    build_tables(ref, w)
    build_tables(lib, w)
    tables, ctx = lib.export(list(range(8)))
    for s in range(8):
        assert tables[s, :4096].tolist() == ref.block_table(s)
    assert ref.num_free() == 0 and lib.num_free() == 0


FAKE = 0x7000_0000  # aligned host address never dereferenced: validation fails first


def _decode_args(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, bt=FAKE, ctx=FAKE, B=4, Hq=8, Hkv=2, D=128, BS=16, NB=64,
             MBS=8, scale=0.1, dtype=binding.PA_BF16, out=FAKE, err=None, stream=None)
    a.update(over)
    return a


def _call_decode(a):
    lib = binding.library()
    return lib.pa_decode(a["q"], a["k"], a["v"], a["bt"], a["ctx"], a["B"], a["Hq"], a["Hkv"],
                         a["D"], a["BS"], a["NB"], a["MBS"], a["scale"], a["dtype"], a["out"],
                         a["err"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(q=None), binding.PA_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), binding.PA_ERR_INVALID_ARG),
    (dict(dtype=7), binding.PA_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), binding.PA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.PA_ERR_INVALID_ARG),
    (dict(NB=1 << 30), binding.PA_ERR_INVALID_ARG),
    (dict(D=96), binding.PA_ERR_UNSUPPORTED),
    (dict(BS=8), binding.PA_ERR_UNSUPPORTED),
    (dict(Hq=64, Hkv=2), binding.PA_ERR_UNSUPPORTED),
    (dict(dtype=binding.PA_F32, Hq=6, Hkv=2), binding.PA_ERR_UNSUPPORTED),
    (dict(dtype=binding.PA_F32, D=256, Hq=2), binding.PA_ERR_UNSUPPORTED),
])
def test_decode_rejects_bad_arguments(over, status):
    assert _call_decode(_decode_args(**over)) == status
    assert binding.library().pa_last_error_string() != b""


def test_split_workspace_size():
    lib = binding.library()
    n = lib.pa_decode_split_workspace_size(8, 64, 128, 16, 8193, 512)
    pmax = -(-8193 // 32)
    rows = 8 * 64 * pmax
    assert n >= 256 + rows * 4 * 2 + rows * 128 * 4
    assert n % 256 == 0
    assert lib.pa_decode_split_workspace_size(8, 64, 128, 16, 100, 500) == 0  # not a multiple


def test_append_and_copy_reject_bad_arguments():
    lib = binding.library()
    assert lib.pa_kv_append(FAKE, FAKE, FAKE, 4, 2, 128, 16, 8, 9, FAKE, FAKE, None, None) == \
        binding.PA_ERR_INVALID_ARG
    assert lib.pa_kv_append(FAKE, FAKE, None, 4, 2, 128, 16, 8, binding.PA_BF16, FAKE, FAKE, None,
                            None) == binding.PA_ERR_INVALID_ARG
    assert lib.pa_kv_append(FAKE, FAKE, FAKE, 0, 2, 128, 16, 8, binding.PA_BF16, FAKE, FAKE, None,
                            None) == binding.PA_OK  # nothing to do
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 3, 100, 8, None, None) == binding.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 0, 4096, 8, None, None) == binding.PA_OK


def test_block_manager_rejects_bad_arguments():
    with pytest.raises(InvalidArgumentError):
        LibBM(3, 4, 2, [0, 0, 1])
    bm = LibBM(4, 4, 2)
    with pytest.raises(InvalidArgumentError):
        bm.allocate(0, 9)
    bm.allocate(0, 8)
    with pytest.raises(InvalidArgumentError):
        bm.append_slot(0)
    with pytest.raises(InvalidArgumentError):
        bm.fork(5, 6)
    with pytest.raises(InvalidArgumentError):
        bm.append_slots([0, 0])
    with pytest.raises(PagedKVError):
        bm.refcount_of(99)


def test_decode_step_rejects_before_touching_the_device():
    import ctypes
    lib = binding.library()
    bm = LibBM(2, 4, 2, [0, 1])
    bm.allocate(7, 8)                       # two full blocks: the next append needs a third
    b = binding.StepBuffers()
    b.max_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim = 2, 2, 2, 64
    b.block_size, b.num_blocks, b.max_blocks_per_seq = 4, 2, 2
    b.partition_tokens, b.scale, b.dtype = 4, 0.1, binding.PA_BF16
    for name in ("k_pool", "v_pool", "workspace", "d_q", "d_k_new", "d_v_new", "d_out",
                 "d_slots", "d_pairs", "d_tables", "d_context_lens"):
        setattr(b, name, FAKE)
    host = {n: np.zeros(16, dtype=np.int64) for n in ("h_slots", "h_pairs", "h_tables", "h_context_lens")}
    for n, a in host.items():
        setattr(b, n, a.ctypes.data)
    ids = np.array([7], dtype=np.int64)
    ncow = ctypes.c_int(-1)
    args = (FAKE, FAKE, FAKE, FAKE, ctypes.byref(ncow), 1, None, None)
    # more sequences than the staging holds
    assert lib.pa_decode_step(bm._h, ctypes.byref(b), np.zeros(3, np.int64).ctypes.data, 3, *args) == \
        binding.PA_ERR_INVALID_ARG
    # block manager failure: reported, nothing changed, nothing enqueued
    before = (bm.block_table(7), bm.context_len(7), bm.free_queue_list())
    assert lib.pa_decode_step(bm._h, ctypes.byref(b), ids.ctypes.data, 1, *args) == \
        binding.PA_ERR_INVALID_ARG          # at max_blocks_per_seq
    assert (bm.block_table(7), bm.context_len(7), bm.free_queue_list()) == before
    bm2 = LibBM(2, 4, 4, [0, 1])
    bm2.allocate(7, 8)
    assert lib.pa_decode_step(bm2._h, ctypes.byref(b), ids.ctypes.data, 1, *args) == \
        binding.PA_ERR_NO_FREE_BLOCKS
    assert bm2.context_len(7) == 8 and bm2.free_queue_list() == []
    assert ctypes.sizeof(binding.StepBuffers) == 208
    # a copy stream without its events is rejected before the manager step
    b.copy_stream = FAKE
    assert lib.pa_decode_step(bm2._h, ctypes.byref(b), ids.ctypes.data, 1, *args) == \
        binding.PA_ERR_INVALID_ARG
    assert bm2.context_len(7) == 8
    b.copy_stream = None


def _reference_groups(tables_by_pos, ctx_by_pos, bs, min_shared=1):
    """Independent statement of the grouping: bucket by first block in batch
    order; shared = longest common table prefix, capped at blocks full for all."""
    buckets, order = {}, []
    for i, t in enumerate(tables_by_pos):
        if not t:
            continue
        if t[0] not in buckets:
            buckets[t[0]] = []
            order.append(t[0])
        buckets[t[0]].append(i)
    offs, members, blocks = [0], [], []
    for b0 in order:
        mem = buckets[b0]
        if len(mem) < 2:
            continue
        shared = min(ctx_by_pos[i] // bs for i in mem)
        for i in mem:
            k = 0
            while k < shared and tables_by_pos[i][k] == tables_by_pos[mem[0]][k]:
                k += 1
            shared = k
        if shared < max(1, min_shared):
            continue
        members += mem
        blocks.append(shared)
        offs.append(len(members))
    return offs, members, blocks


@pytest.mark.parametrize("name", ["prefix", "prefix_cow", "tiny", "gqa"])
def test_prefix_groups_match_reference(name):
    w = workloads.WORKLOADS[name]()
    bm = LibBM(w.num_blocks, w.block_size, w.max_blocks_per_seq, w.free_order)
    build_tables(bm, w)
    if w.step_seqs:
        bm.append_slots_arrays(w.step_seqs)
    seqs = list(w.decode_seqs)
    rng = np.random.default_rng(3)
    rng.shuffle(seqs)
    offs, members, blocks = bm.prefix_groups(seqs)
    tabs = [bm.block_table(s) for s in seqs]
    ctxs = [bm.context_len(s) for s in seqs]
    want = _reference_groups(tabs, ctxs, w.block_size)
    assert (offs.tolist(), members.tolist(), blocks.tolist()) == want
    if name.startswith("prefix"):
        assert len(blocks) == 8 and all(b == 250 for b in blocks)
        assert all(offs[g + 1] - offs[g] == 16 for g in range(8))
    if name == "gqa":
        assert len(blocks) == 0   # no sharing


def test_prefix_groups_partial_sharing_and_threshold():
    bm = LibBM(40, 4, 10, list(range(40)))
    bm.allocate(0, 17)          # blocks 0..4, tail holds 1 token
    bm.fork(0, 1)
    bm.fork(0, 2)
    for _ in range(3):
        bm.append_slot(1)       # 1 copies block 4 on its first append
    bm.allocate(3, 8)
    offs, members, blocks = bm.prefix_groups([3, 2, 1, 0])
    assert offs.tolist() == [0, 3] and members.tolist() == [1, 2, 3] and blocks.tolist() == [4]
    offs, members, blocks = bm.prefix_groups([3, 2, 1, 0], min_shared_blocks=5)
    assert offs.tolist() == [0] and members.size == 0


def test_shared_prefix_rejects_bad_groups_on_host():
    lib = binding.library()
    a = _decode_args()
    base = [a["q"], a["k"], a["v"], a["bt"], a["ctx"], a["B"], a["Hq"], a["Hkv"], a["D"], a["BS"],
            a["NB"], a["MBS"], a["scale"], a["dtype"], 512]
    ws = FAKE

    def call(offs, members, blocks, ng):
        o = np.asarray(offs, np.int32); m = np.asarray(members, np.int32); b = np.asarray(blocks, np.int32)
        return lib.pa_decode_shared_prefix(*base, ng, o.ctypes.data, m.ctypes.data, b.ctypes.data,
                                           ws, 1 << 40, a["out"], None, None)
    assert call([0, 2], [0, 0], [1], 1) == binding.PA_ERR_INVALID_ARG      # repeated member
    assert call([0, 2], [0, 9], [1], 1) == binding.PA_ERR_INVALID_ARG      # member past the batch
    assert call([1, 2], [0, 1], [1], 1) == binding.PA_ERR_INVALID_ARG      # offsets start at 1
    assert call([0, 2], [0, 1], [99], 1) == binding.PA_ERR_INVALID_ARG     # more blocks than the table
    base[13] = binding.PA_F32
    assert call([0, 2], [0, 1], [1], 1) == binding.PA_ERR_UNSUPPORTED      # bf16 only


def test_nvtx_ranges_compile_in_only_with_the_build_flag(tmp_path):
    """With PAGEDKV_NVTX defined (build.py --nvtx) the C-ABI sources carry
    NVTX ranges around the calls that enqueue GPU work; the default build
    references no NVTX symbol."""
    import subprocess
    from paged_kv_cache_336_b200 import build as B
    src = os.path.join(B.CSRC, "step_api.cu")
    syms = {}
    for variant, defines in (("plain", ()), ("nvtx", ("PAGEDKV_NVTX=1",))):
        obj = str(tmp_path / f"step_{variant}.o")
        B._compile(src, obj, False, defines)
        syms[variant] = subprocess.run(["nm", obj], capture_output=True, text=True,
                                       check=True).stdout
    assert "nvtxRangePushA" in syms["nvtx"] or "nvtxGlobals" in syms["nvtx"]
    assert "nvtx" not in syms["plain"].lower()
    # every C entry point that launches work opens a range
    for name, path in (("pa_decode", "decode_api.cu"), ("pa_decode_split", "decode_api.cu"),
                       ("pa_decode_split_static", "decode_api.cu"),
                       ("pa_decode_shared_prefix", "decode_api.cu"),
                       ("pa_decode_split_window", "decode_api.cu"), ("pa_prefill", "decode_api.cu"),
                       ("pa_kv_append", "kv_ops.cu"), ("pa_copy_blocks", "kv_ops.cu"),
                       ("pa_swap_out", "kv_ops.cu"), ("pa_swap_in", "kv_ops.cu"),
                       ("pa_decode_step", "step_api.cu")):
        text = open(os.path.join(B.CSRC, path)).read()
        assert f'PA_NVTX_RANGE("{name}");' in text, name
