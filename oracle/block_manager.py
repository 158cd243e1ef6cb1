"""Reference host block manager (test infrastructure).

What it does, with the passage each rule follows:

* Each sequence owns logical blocks 0..n-1 and a block table mapping them to
  physical block IDs; prefill reserves enough blocks for the input; decode
  appends into the partly filled tail and takes a new block only when the
  tail is full ("What is PagedAttention?", How It Works / Map Logical to
  Physical Blocks).
* An allocation that cannot be met is reported explicitly and must not
  disturb any sequence's state (same passage). Here every call is
  all-or-nothing: on failure nothing changes.
* Sequences share blocks by pointing their tables at the same physical
  blocks; a per-block reference count is incremented and nothing is copied
  ("PagedAttention: Optimizing KV Cache in vLLM", section 4, step 1).
* Before writing into a block whose count is above one, the writer gets a
  new block, the contents are copied, and only the writer's table changes
  (same section, steps 2-3; "What is PagedAttention?", Share Without
  Mutating State). The shared block's count drops by one.
* Blocks whose count reaches zero go back to the free pool (reference counts
  govern reclamation).

Policy choices the pages leave open (each is the plainest reading):

* Free blocks form a FIFO queue, seeded from ``initial_free_order``
  (identity when omitted). Allocation pops from the front; a ``free`` call
  pushes the blocks it reclaims to the back in ascending block-ID order.
* A copy-on-write copies the whole block (all heads, all slots). One page
  says the copy covers the block's valid entries, another that it covers the
  shared block's contents; the whole block covers both.
* ``append_slots`` processes sequences in the order given. A shared partial
  tail is copied by each writer while its count is above one; the last
  holder (count one) writes in place.
"""

from __future__ import annotations

from collections import deque
from dataclasses import dataclass


class InvalidArgument(ValueError):
    """Unknown or duplicate sequence, capacity of a block table exceeded, ..."""


class NoFreeBlocks(RuntimeError):
    """The free pool cannot satisfy the request; no state was changed."""


@dataclass
class AppendResult:
    slot: int
    cow_src: int = -1
    cow_dst: int = -1


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, max_blocks_per_seq: int,
                 initial_free_order=None):
        if num_blocks <= 0 or block_size <= 0 or max_blocks_per_seq <= 0:
            raise InvalidArgument("sizes must be positive")
        if initial_free_order is None:
            order = list(range(num_blocks))
        else:
            order = [int(b) for b in initial_free_order]
            if sorted(order) != list(range(num_blocks)):
                raise InvalidArgument("initial_free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_blocks_per_seq = max_blocks_per_seq
        self.free_queue = deque(order)
        self.refcount = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.context: dict[int, int] = {}
        self.swapped: dict[int, list[int]] = {}   # table at swap-out time
        self.cow_copies = 0

    # -- queries -----------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free_queue)

    def block_table(self, seq: int) -> list[int]:
        self._require(seq)
        return list(self.tables[seq])

    def context_len(self, seq: int) -> int:
        self._require(seq)
        return self.context[seq]

    def stats(self) -> dict:
        used = sum(1 for rc in self.refcount if rc > 0)
        shared = sum(1 for rc in self.refcount if rc > 1)
        # resident blocks and tokens (a released window prefix no longer counts)
        resident = {s: sum(1 for b in t if b >= 0) for s, t in self.tables.items()}
        logical_slots = sum(resident.values()) * self.block_size
        tokens = sum(0 if s in self.swapped else
                     ctx - (len(self.tables[s]) - resident[s]) * self.block_size
                     for s, ctx in self.context.items())
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": len(self.free_queue),
            "used_blocks": used,
            "shared_blocks": shared,
            "num_seqs": len(self.tables),
            "logical_tokens": tokens,
            "logical_slots": logical_slots,
            "tail_waste_slots": logical_slots - tokens,
            "cow_copies": self.cow_copies,
        }

    # -- operations ----------------------------------------------------------
    def allocate(self, seq: int, num_tokens: int) -> None:
        """Prefill: reserve ceil(num_tokens / block_size) blocks, all or nothing."""
        if seq in self.tables:
            raise InvalidArgument(f"sequence {seq} already exists")
        if num_tokens < 0:
            raise InvalidArgument("num_tokens must be >= 0")
        need = -(-num_tokens // self.block_size)
        if need > self.max_blocks_per_seq:
            raise InvalidArgument("sequence exceeds max_blocks_per_seq")
        if need > len(self.free_queue):
            raise NoFreeBlocks(f"need {need} blocks, {len(self.free_queue)} free")
        table = [self.free_queue.popleft() for _ in range(need)]
        for b in table:
            self.refcount[b] = 1
        self.tables[seq] = table
        self.context[seq] = num_tokens

    def fork(self, parent: int, child: int) -> None:
        """Child shares all of the parent's blocks; counts go up, no data moves."""
        self._require(parent)
        if parent in self.swapped:
            raise InvalidArgument(f"sequence {parent} is swapped out")
        if child in self.tables:
            raise InvalidArgument(f"sequence {child} already exists")
        table = list(self.tables[parent])
        for b in table:
            if b >= 0:
                self.refcount[b] += 1
        self.tables[child] = table
        self.context[child] = self.context[parent]

    def _need_for_append(self, seq: int, refcount_view) -> int:
        if seq in self.swapped:
            raise InvalidArgument(f"sequence {seq} is swapped out")
        ctx = self.context[seq]
        table = self.tables[seq]
        if ctx % self.block_size == 0:
            if len(table) >= self.max_blocks_per_seq:
                raise InvalidArgument(f"sequence {seq} is at max_blocks_per_seq")
            return 1
        tail = table[-1]
        return 1 if refcount_view[tail] > 1 else 0

    def append_slot(self, seq: int) -> AppendResult:
        """Reserve the slot for one new token of ``seq`` (decode step)."""
        return self.append_slots([seq])[0]

    def append_slots(self, seqs) -> list[AppendResult]:
        """One decode step for several sequences, all or nothing, in order."""
        seqs = [int(s) for s in seqs]
        if len(set(seqs)) != len(seqs):
            raise InvalidArgument("duplicate sequence in one step")
        for s in seqs:
            self._require(s)
        # Dry run on a scratch view of the counts to learn how many blocks the
        # step needs; earlier copy-on-writes lower the counts later writers see.
        rc = {}
        need = 0
        for s in seqs:
            view = _Overlay(self.refcount, rc)
            n = self._need_for_append(s, view)
            if n and self.context[s] % self.block_size != 0:
                tail = self.tables[s][-1]
                rc[tail] = view[tail] - 1
            need += n
        if need > len(self.free_queue):
            raise NoFreeBlocks(f"step needs {need} blocks, {len(self.free_queue)} free")
        return [self._append_one(s) for s in seqs]

    def _append_one(self, seq: int) -> AppendResult:
        ctx = self.context[seq]
        table = self.tables[seq]
        offset = ctx % self.block_size
        result = AppendResult(slot=-1)
        if offset == 0:
            block = self.free_queue.popleft()
            self.refcount[block] = 1
            table.append(block)
        else:
            block = table[-1]
            if self.refcount[block] > 1:
                new_block = self.free_queue.popleft()
                self.refcount[new_block] = 1
                self.refcount[block] -= 1
                table[-1] = new_block
                result.cow_src, result.cow_dst = block, new_block
                self.cow_copies += 1
                block = new_block
        result.slot = block * self.block_size + offset
        self.context[seq] = ctx + 1
        return result

    def release_before(self, seq: int, first_token: int) -> list[int]:
        """Sliding window: drop this sequence's references to blocks whose
        tokens all lie before ``first_token``; their table entries become -1
        (logical positions are kept). Returns the blocks reclaimed (count 0),
        which go to the back of the free queue in ascending order."""
        self._require(seq)
        if first_token < 0:
            raise InvalidArgument("first_token must be >= 0")
        if seq in self.swapped:
            raise InvalidArgument(f"sequence {seq} is swapped out")
        table = self.tables[seq]
        n_out = min(first_token // self.block_size, len(table))
        reclaimed = []
        for i in range(n_out):
            b = table[i]
            if b < 0:
                continue
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                reclaimed.append(b)
            table[i] = -1
        for b in sorted(reclaimed):
            self.free_queue.append(b)
        return sorted(reclaimed)

    def swap_out(self, seq: int) -> list[int]:
        """Preemption by swapping ("What is PagedAttention?", How It Works:
        an allocation failure is met by admission control, preemption, swap
        or rejection). The sequence keeps its context length but gives up
        its blocks: every resident table entry's count drops by one (blocks
        reaching zero are reclaimed, ascending, to the back of the queue).
        Returns the blocks in table order (-1 for released entries): the
        caller copies them to host memory before the pool reuses them."""
        self._require(seq)
        if seq in self.swapped:
            raise InvalidArgument(f"sequence {seq} is already swapped out")
        table = self.tables[seq]
        reclaimed = []
        for b in table:
            if b < 0:
                continue
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                reclaimed.append(b)
        for b in sorted(reclaimed):
            self.free_queue.append(b)
        self.swapped[seq] = list(table)
        self.tables[seq] = [-1 if b >= 0 else b for b in table]
        return list(table)

    def swap_in(self, seq: int) -> list[int]:
        """Bring a swapped-out sequence back: one new private block per
        previously resident entry, popped from the queue in table order, all
        or nothing. Returns the new table (the caller copies the host copies
        into the new blocks)."""
        self._require(seq)
        if seq not in self.swapped:
            raise InvalidArgument(f"sequence {seq} is not swapped out")
        old = self.swapped[seq]
        need = sum(1 for b in old if b >= 0)
        if need > len(self.free_queue):
            raise NoFreeBlocks(f"swap-in needs {need} blocks, {len(self.free_queue)} free")
        table = []
        for b in old:
            if b < 0:
                table.append(b)
            else:
                nb = self.free_queue.popleft()
                self.refcount[nb] = 1
                table.append(nb)
        self.tables[seq] = table
        del self.swapped[seq]
        return list(table)

    def free(self, seq: int) -> None:
        """Drop a finished sequence; reclaim blocks whose count reaches zero."""
        self._require(seq)
        reclaimed = []
        for b in self.tables[seq]:
            if b < 0:
                continue
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                reclaimed.append(b)
        for b in sorted(reclaimed):
            self.free_queue.append(b)
        del self.tables[seq]
        del self.context[seq]
        self.swapped.pop(seq, None)

    def _require(self, seq: int) -> None:
        if seq not in self.tables:
            raise InvalidArgument(f"unknown sequence {seq}")

    # -- state snapshot (for equality checks in tests) -----------------------
    def snapshot(self) -> tuple:
        return (
            tuple(self.free_queue),
            tuple(self.refcount),
            tuple(sorted((s, tuple(t)) for s, t in self.tables.items())),
            tuple(sorted(self.context.items())),
            self.cow_copies,
        )

    def is_swapped(self, seq: int) -> bool:
        self._require(seq)
        return seq in self.swapped


class _Overlay:
    """Read-through view of the counts with a few entries overridden."""

    def __init__(self, base, over):
        self.base = base
        self.over = over

    def __getitem__(self, b):
        return self.over.get(b, self.base[b])
