"""A CPU model of how the balanced split decode cuts a batch into pieces
(paged_decode_stream_kernel), checked before any GPU run and kept as a test.

Each KV head's work is one list of 16-token units, sequence after sequence.
Global warp w works for KV head w % Hkv in group w // Hkv and takes units
[g*C, (g+1)*C) of that head's list, with groups = warps // Hkv and
C = max(ceil(U / groups), ceil(U_max / (P - 1))), where U_max is the most
units any sequence has and P the most pieces the workspace holds per
(sequence, KV head), ceil(max_blocks_per_seq / (partition_tokens /
block_size)) + 1. A (sequence, KV head) is a segment; the warp holding its
first unit records its number of pieces, and every warp writes its piece of
a segment to partial slot base + piece. The model below restates those rules
and checks, over random batches (empty sequences, windows, shared-prefix
skips, block sizes 16 and 32, tiny and large grids), that:

* every unit of every KV head is taken by exactly one warp, in order;
* the pieces of a segment are numbered 0 .. pieces-1, one per warp that
  touches it, and only a segment held whole by one warp is written as a
  final output;
* pieces never exceed P, so base + piece stays inside the row's slots.
"""

import math

import numpy as np
import pytest


def first_unit(ctx, bs, window, skip_blocks):
    ub = (max(0, ctx - window) if window > 0 and ctx > window else 0) // 16
    if skip_blocks is not None:
        ub = max(ub, min(max(skip_blocks, 0), ctx // bs) * (bs // 16))
    ue = (ctx + 15) // 16
    return ub if ub < ue else -1


def decompose(ctx, hkv, bs, window, skips, nwarps, max_pieces):
    ub = [first_unit(int(c), bs, window, None if skips is None else int(skips[s]))
          for s, c in enumerate(ctx)]
    units = [1 if u < 0 else (int(c) + 15) // 16 - u for u, c in zip(ub, ctx)]
    prefix = np.concatenate([[0], np.cumsum(units)]).astype(np.int64)
    U = int(prefix[-1])
    groups = nwarps // hkv
    assert groups >= 1
    C = max(-(-U // groups), -(-max(units) // (max_pieces - 1)))
    writes = []   # (warp, s, kvh, first unit in segment, last+1, piece, whole)
    pieces = {}
    for w in range(nwarps):
        h, gi = w % hkv, w // hkv
        if gi >= groups:
            continue
        g0, g1 = min(gi * C, U), min((gi + 1) * C, U)
        if g1 <= g0:
            continue
        s = int(np.searchsorted(prefix, g0, side="right") - 1)
        us = units[s]
        un = g0 - int(prefix[s])
        seg_start = g0 - un
        start_un = un
        g = g0
        while g < g1:
            if un == us:
                writes.append((w, s, h, start_un, un, gi - seg_start // C, seg_start >= g0))
                seg_start += us
                s += 1
                us = units[s]
                un = start_un = 0
            if un == 0:
                assert (s, h) not in pieces
                pieces[(s, h)] = (seg_start + us - 1) // C - seg_start // C + 1
            un += 1
            g += 1
        writes.append((w, s, h, start_un, un, gi - seg_start // C, un == us and seg_start >= g0))
    return units, writes, pieces, C


@pytest.mark.parametrize("seed", range(40))
def test_every_unit_once_and_pieces_fit_the_workspace(seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([16, 32]))
    hkv = int(rng.choice([1, 2, 8]))
    B = int(rng.integers(1, 40))
    mbs = int(rng.integers(1, 300))
    ctx = rng.integers(0, mbs * bs + 1, size=B)
    ctx[rng.random(B) < 0.1] = 0
    window = int(rng.choice([0, 0, 1, 7, 100, 4096]))
    shared = rng.random() < 0.3
    skips = rng.integers(0, mbs + 1, size=B) if shared else None
    base_slots = 16 if shared else 0
    ptok = bs * int(rng.integers(1, 40))
    nwarps = max(hkv, int(rng.choice([1, 3, 8, 148 * 8, 1184, 1776])))
    max_pieces = math.ceil(mbs / (ptok // bs)) + 1
    units, writes, pieces, C = decompose(ctx, hkv, bs, window, skips, nwarps, max_pieces)
    pmax = max_pieces + base_slots

    # coverage: the writes tile every segment's units exactly, in order
    seen = {}
    for w, s, kvh, a, b, piece, whole in writes:
        seen.setdefault((s, kvh), []).append((a, b, piece, whole, w))
    assert set(seen) == {(s, k) for s in range(B) for k in range(hkv)}
    for (s, kvh), parts in seen.items():
        parts.sort()
        assert parts[0][0] == 0 and parts[-1][1] == units[s]
        for (a0, b0, *_), (a1, *_) in zip(parts, parts[1:]):
            assert b0 == a1
        # pieces numbered 0.. in warp order, one per warp; count recorded once
        assert [p[2] for p in parts] == list(range(len(parts)))
        assert pieces[(s, kvh)] == len(parts)
        assert [p[4] for p in parts] == sorted(p[4] for p in parts)
        # a final output only when one warp holds the whole segment
        assert any(p[3] for p in parts) == (len(parts) == 1)
        # slots stay inside the row
        assert len(parts) <= max_pieces and base_slots + len(parts) - 1 < pmax
        # the warps of a piece list all work for the segment's KV head
        assert all(p[4] % hkv == kvh for p in parts)


def test_balance_long_context_batch():
    """The measured long-context batch: 8 x 131072 tokens, 8 KV heads, block
    16, 512-token partitions (at most 258 pieces), 444 CTAs x 4 warps: every
    warp but the last group's streams exactly C = ceil(U / groups) units (the
    last group the rest), and each segment has about 30 pieces."""
    ctx = np.full(8, 131072)
    mbs = 131072 // 16 + 64
    units, writes, pieces, C = decompose(ctx, 8, 16, 0, None, 1776, math.ceil(mbs / 32) + 1)
    per_warp = {}
    for w, s, kvh, a, b, *_ in writes:
        per_warp[w] = per_warp.get(w, 0) + (b - a)
    U = 8 * 8192                                    # units of each KV head's list
    last = (U - 1) // C                             # the last group with work
    for w, n in per_warp.items():
        assert n == (C if w // 8 < last else U - last * C)
    # the busiest warp streams ceil(U / groups) units: under one unit above the mean
    assert last == 1776 // 8 - 1 and C == -(-U // (1776 // 8))
    assert max(pieces.values()) <= 31


def test_many_one_unit_sequences_spread_over_warps():
    """Shared-prefix suffixes: 128 sequences of one unit each, 8 KV heads,
    long tables: one unit per warp (the piece bound does not force long
    chunks when every segment is short)."""
    units, writes, pieces, C = decompose(np.full(128, 5), 8, 16, 0, None, 1776, 260)
    assert C == 1
    assert len({w for w, *_ in writes}) == 128 * 8
