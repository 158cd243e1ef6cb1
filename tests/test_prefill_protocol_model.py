"""A discrete-event model of the persistent tcgen05 prefill kernel's
hand-over protocol (csrc/tc_prefill_kernel.cuh), run on the CPU.

Each CTA role is a generator that follows the kernel's loops and running
counts: the producer (K/V ring, partial-chunk V clears), the two MMA
issuers (Q copies, S and P V MMAs, commits) and the two tiles' softmax
warps (P, epilogue), two per tile since each row's 64 logits are split
between two threads of different warps: the halves swap their row maxima
every chunk (and their row sums at an item's end) through a double-buffered
exchange completed by an mbarrier. Barriers count arrivals and completed phases as
mbarriers do. TMA copies and tensor-core work finish after random delays.
MMAs are ordered only where tcgen05 orders them: those accumulating into the
same TMEM region run in issue order; others may overlap or overtake one
another. A commit arrives once all of its thread's earlier MMAs are done.

A kernel wait only knows a parity, so it is right only while the barrier
has completed the phase it means or the one before it. The model checks that
at every poll (no wait early by a phase, none lapped), that no role
deadlocks, and that no buffer is overwritten while in use: a ring slot is
refilled only after every MMA reading its last use has finished; an S MMA
starts only after the softmax is done with the buffer's previous chunk and
that chunk's P V has read its P; Q, O and a partial chunk's cleared V rows
likewise. Random item lists mix idle second tiles, empty spans, one-chunk
items and partial last chunks. The last tests plant each guard's absence and
expect the model to catch it."""

import heapq
import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.n = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: more arrivals than expected"
        if self.pending == 0:
            self.n += 1
            self.pending = self.count


def simulate(items, nslot, tiles, seed, tail_guard=True, q_free_wait=True, s_waits_p_free=True,
             exchange_wait=True):
    """items: (chunks, active tiles, partial last chunk) per item, in one
    CTA's order. Returns None, or a description of the first fault."""
    rnd = random.Random(seed)
    kv_full = [Bar(f"kv_full{i}", 1) for i in range(nslot)]
    kv_empty = [Bar(f"kv_empty{i}", tiles) for i in range(nslot)]
    s_full = [Bar(f"s_full{i}", 1) for i in range(4)]
    p_full = [Bar(f"p_full{i}", 8) for i in range(4)]
    p_free = [Bar(f"p_free{i}", 1) for i in range(4)]
    q_full = [Bar(f"q_full{i}", 1) for i in range(2)]
    q_free = [Bar(f"q_free{i}", 1) for i in range(2)]
    o_last = [Bar(f"o_last{i}", 1) for i in range(2)]
    o_empty = [Bar(f"o_empty{i}", 8) for i in range(2)]
    mma_done = [Bar(f"mma_done{i}", 1) for i in range(2)]
    v_tail = Bar("v_tail", 1)
    # the two halves of a tile's softmax swap their row maxima (and, at an
    # item's end, their row sums) through a double-buffered exchange; one
    # arrival here stands for the 128 threads of a half
    xchg = [Bar(f"xchg{i}", 2) for i in range(4)]
    xval = {}                          # (tile, buffer, half) -> (exchange written, read yet)

    now = [0]
    events, seq = [], [0]
    last_of = {}
    s_end, o_read = {}, {}
    slot_read_end = {}                 # ring slot -> end of the last MMA reading it
    sm_done, pv_end = {}, {}           # (tile, chunk[, half]) -> softmax finished / its P V ended
    s_read = {}                        # (tile, chunk, half) -> that half read its logits
    tail_cleared = {}                  # ring index of a partial chunk's V -> time cleared
    faults = []

    def reads_slot(slot, end):
        slot_read_end[slot] = max(slot_read_end.get(slot, 0), end)

    def later(t, bar):
        seq[0] += 1
        heapq.heappush(events, (t, seq[0], bar))

    acc_end = {}

    def mma(tid, dur, acc):
        start = max(acc_end.get(acc, 0), now[0]) + rnd.randint(0, 300)
        end = start + dur
        acc_end[acc] = end
        last_of[tid] = max(last_of.get(tid, 0), end)
        return start, end

    def commit(tid, bar):
        later(max(last_of.get(tid, 0), now[0]) + 1, bar)

    def wait(bar, phase):
        return ("wait", bar, phase)

    def producer():
        g, prev_tail = 0, -1
        for nch, _, tail in items:
            if nch == 0:
                continue
            for i in range(2 * nch):
                gi = g + i
                if gi >= nslot:
                    yield wait(kv_empty[gi % nslot], gi // nslot - 1)
                if now[0] < slot_read_end.get(gi % nslot, 0):
                    faults.append(f"slot {gi % nslot} refilled while an MMA still reads it")
                later(now[0] + rnd.randint(50, 3000), kv_full[gi % nslot])
                yield ("delay", rnd.randint(5, 60))
            if tail:
                gi = g + 2 * nch - 1
                yield wait(kv_full[gi % nslot], gi // nslot)
                if tail_guard and prev_tail >= 0 and gi - prev_tail < nslot:
                    yield wait(kv_empty[prev_tail % nslot], prev_tail // nslot)
                yield ("delay", 100)
                tail_cleared[gi] = now[0]
                v_tail.arrive()
                prev_tail = gi
            g += 2 * nch
        for gi in range(max(0, g - nslot), g):
            yield wait(kv_full[gi % nslot], gi // nslot)

    def issuer(t):
        tid = ("issuer", t)
        g = cb = nt = tails = 0
        q_loads, q_seen = [0], [0]

        def load_q():
            if now[0] < s_end.get(t, 0):
                faults.append(f"tile {t}: Q overwritten before the last S read it")
            later(now[0] + rnd.randint(200, 3000), q_full[t])
            q_loads[0] += 1

        for idx, (nch, ntiles, tail) in enumerate(items):
            if nch == 0:
                continue
            if t >= ntiles:
                for i in range(2 * nch):
                    gi = g + i
                    yield wait(kv_full[gi % nslot], gi // nslot)
                    kv_empty[gi % nslot].arrive()
                g += 2 * nch
                tails += 1 if tail else 0
                continue
            if q_loads[0] == q_seen[0]:
                load_q()
            yield wait(q_full[t], q_seen[0])
            q_seen[0] += 1

            def issue_s(j):
                gi, c = g + 2 * j, cb + j
                yield wait(kv_full[gi % nslot], gi // nslot)
                if c >= 2 and s_waits_p_free:
                    yield wait(p_free[2 * t + (c & 1)], (c >> 1) - 1)
                start, end = mma(tid, rnd.randint(200, 500), ("S", t, c & 1))
                done = max(sm_done.get((t, c - 2, h), 1 << 60) for h in (0, 1))
                if c >= 2 and start < max(done, pv_end.get((t, c - 2), 1 << 60)):
                    faults.append(f"tile {t}: S({c}) overwrote a buffer still in use for chunk {c - 2}")
                reads_slot(gi % nslot, end)
                s_end[t] = max(s_end.get(t, 0), end)
                commit(tid, s_full[2 * t + (c & 1)])
                commit(tid, kv_empty[gi % nslot])

            def after_last_s():
                commit(tid, q_free[t])
                for n in range(idx + 1, len(items)):
                    if items[n][0] == 0 or t >= items[n][1]:
                        continue
                    if q_free_wait:
                        yield wait(q_free[t], nt)
                    load_q()
                    break

            yield from issue_s(0)
            if nch == 1:
                yield from after_last_s()
            for j in range(nch):
                if j + 1 < nch:
                    yield from issue_s(j + 1)
                    if j + 2 == nch:
                        yield from after_last_s()
                gi, c = g + 2 * j + 1, cb + j
                yield wait(kv_full[gi % nslot], gi // nslot)
                if tail and j == nch - 1:
                    yield wait(v_tail, tails)
                yield wait(p_full[2 * t + (c & 1)], c >> 1)
                if j == 0 and nt > 0:
                    yield wait(o_empty[t], nt - 1)
                start, end = mma(tid, rnd.randint(150, 400), ("O", t))
                if j == 0 and nt > 0 and start < max(o_read[(t, nt - 1, h)] for h in (0, 1)):
                    faults.append(f"tile {t}: O overwritten before the epilogue read it")
                if tail and j == nch - 1 and start < tail_cleared.get(gi, 1 << 60):
                    faults.append(f"tile {t}: P V read a partial chunk's V before it was cleared")
                pv_end[(t, c)] = end
                reads_slot(gi % nslot, end)
                commit(tid, p_free[2 * t + (c & 1)])
                commit(tid, kv_empty[gi % nslot])
            commit(tid, o_last[t])
            g += 2 * nch
            cb += nch
            tails += 1 if tail else 0
            nt += 1
        if q_loads[0] > q_seen[0]:
            yield wait(q_full[t], q_seen[0])
        commit(tid, mma_done[t])
        yield wait(mma_done[t], 0)

    def softmax(t, hf):
        cb = nt = ex = 0
        other = 1 - hf

        def exchange():
            nonlocal ex
            b = ex & 1
            prev = xval.get((t, b, hf))
            if prev is not None and not prev[1]:
                faults.append(f"tile {t} half {hf}: exchange {ex} overwrites exchange {prev[0]} "
                              f"before the other half read it")
            xval[(t, b, hf)] = (ex, False)
            xchg[2 * t + b].arrive()
            if exchange_wait:
                yield wait(xchg[2 * t + b], ex >> 1)
            yield ("delay", rnd.randint(0, 200))
            got = xval.get((t, b, other))
            if got is None or got[0] != ex:
                faults.append(f"tile {t} half {hf}: read {got} at exchange {ex}")
            else:
                xval[(t, b, other)] = (got[0], True)
            ex += 1

        for nch, ntiles, _ in items:
            if t >= ntiles:
                continue
            for j in range(nch):
                c = cb + j
                yield wait(s_full[2 * t + (c & 1)], c >> 1)
                yield ("delay", rnd.randint(100, 500))       # read this half's logits
                s_read[(t, c, hf)] = now[0]
                yield from exchange()                        # row maximum
                yield ("delay", rnd.randint(150, 800))
                if j >= 1 and rnd.random() < 0.1:  # a rescale of O (this half's columns)
                    yield wait(p_free[2 * t + ((c - 1) & 1)], (c - 1) >> 1)
                    if now[0] < pv_end.get((t, c - 1), 1 << 60):
                        faults.append(f"tile {t}: O rescaled while P V({c - 1}) still accumulates")
                    yield ("delay", 100)
                # P is written over the first half of the buffer: the other
                # half's logits there must have been read already
                if s_read.get((t, c, other), 1 << 60) > now[0]:
                    faults.append(f"tile {t} chunk {c}: half {hf} writes P before half {other} "
                                  f"read its logits")
                sm_done[(t, c, hf)] = now[0]
                for _ in range(4):
                    p_full[2 * t + (c & 1)].arrive()
            if nch > 0:
                yield wait(o_last[t], nt)
            yield from exchange()                            # row sums
            yield ("delay", rnd.randint(100, 800))
            if nch > 0:
                o_read[(t, nt, hf)] = now[0]
                for _ in range(4):
                    o_empty[t].arrive()
                cb += nch
                nt += 1

    roles = {"producer": producer(), "issuer0": issuer(0), "softmax0a": softmax(0, 0),
             "softmax0b": softmax(0, 1)}
    if tiles == 2:
        roles.update({"issuer1": issuer(1), "softmax1a": softmax(1, 0), "softmax1b": softmax(1, 1)})
    state = {n: {"gen": g, "wait": None, "wake": 0, "done": False} for n, g in roles.items()}
    while True:
        progressed = True
        while progressed:
            progressed = False
            while events and events[0][0] <= now[0]:
                heapq.heappop(events)[2].arrive()
                progressed = True
            for name, st in state.items():
                if st["done"] or st["wake"] > now[0]:
                    continue
                while True:
                    if st["wait"] is not None:
                        bar, phase = st["wait"]
                        if not phase <= bar.n <= phase + 1:
                            return (f"{name} waits for phase {phase} of {bar.name}, "
                                    f"which has completed {bar.n}")
                        if bar.n == phase:
                            break
                        st["wait"] = None
                    try:
                        act = next(st["gen"])
                    except StopIteration:
                        st["done"] = True
                        progressed = True
                        break
                    progressed = True
                    if act[0] == "wait":
                        st["wait"] = (act[1], act[2])
                    else:
                        st["wake"] = now[0] + act[1]
                        break
        if faults:
            return faults[0]
        if all(st["done"] for st in state.values()):
            return None
        upcoming = [st["wake"] for st in state.values() if not st["done"] and st["wake"] > now[0]]
        if events:
            upcoming.append(events[0][0])
        if not upcoming:
            stuck = {n: (st["wait"][0].name, st["wait"][1]) for n, st in state.items()
                     if not st["done"] and st["wait"]}
            return f"deadlock: {stuck}"
        now[0] = min(upcoming)


def random_items(rnd, tiles):
    items = []
    for _ in range(rnd.randint(1, 12)):
        nch = rnd.choice([0, 1, 1, 2, 3, 5, 9])
        ntiles = min(tiles, rnd.choice([1, 2, 2]))
        items.append((nch, ntiles, nch > 0 and rnd.random() < 0.6))
    return items


@pytest.mark.parametrize("nslot,tiles", [(8, 2), (7, 2), (6, 2), (4, 2), (4, 1)])
def test_protocol_has_no_deadlock_lap_or_overwrite(nslot, tiles):
    for trial in range(250):
        rnd = random.Random(1000 * nslot + 10 * tiles + trial)
        items = random_items(rnd, tiles)
        fault = simulate(items, nslot, tiles, seed=trial)
        assert fault is None, f"trial {trial}, items {items}: {fault}"


def _first_fault(**kw):
    for trial in range(400):
        rnd = random.Random(trial)
        items = random_items(rnd, 2)
        fault = simulate(items, 8, 2, seed=trial, **kw)
        if fault:
            return fault
    return None


def test_model_catches_a_missing_tail_guard():
    fault = _first_fault(tail_guard=False)
    assert fault is not None and "v_tail" in fault


def test_model_catches_a_missing_q_free_wait():
    fault = _first_fault(q_free_wait=False)
    assert fault is not None and "Q overwritten" in fault


def test_model_catches_an_s_mma_that_skips_the_p_free_wait():
    fault = _first_fault(s_waits_p_free=False)
    assert fault is not None and "overwrote a buffer" in fault


def test_model_catches_halves_that_do_not_wait_for_the_exchange():
    fault = _first_fault(exchange_wait=False)
    assert fault is not None and ("read" in fault or "overwrites" in fault or "before half" in fault)
