"""Seeded synthetic inputs for the paged decode path.

This module draws random numbers and fixes shapes; it holds none of the
method's arithmetic (no gather, no softmax, no block-table or slot logic).
Tests feed the same draws to the CUDA path and to the CPU oracle; the bench
uses it to build its workloads.

Workloads (the shapes of the decode configurations this library is measured
on; all values are N(0, 1) draws, all block placements seeded shuffles):

``tiny``    4 sequences, context lengths {1, 15, 16, 33}, block size 16, 2 query
            heads = 2 KV heads, head_dim 64, fp32, pool of 16 blocks whose free
            order is a seeded permutation; then fork(3 -> 4), one appended token
            per sequence 0..3 (sequence 3 copies its shared tail), decode 0..4.
``mha``     batch 64, 32 query heads = 32 KV heads, head_dim 128, bf16, block
            size 16, context lengths uniform in [1, 2048], pool 16384 blocks;
            tables have room for 512 more tokens (bench decode steps).
``gqa``     batch 256, 32 query heads over 8 KV heads, head_dim 128, bf16, block
            size 16, context lengths log-uniform in [16, 8192], pool 110% of the
            blocks needed.
``prefix``  8 prompts of 4000 tokens, each forked into 16 branches; each branch
            then appends 0..512 private tokens; GQA 32/8, head_dim 128, bf16.
``prefix_cow`` the same with 4008-token prompts (250 full blocks plus a shared
            partial block) and no private tokens, so the next appended token of
            every branch but the last lands in a shared partial tail.
``long``    batch 8, context 131072, 64 query heads over 8 KV heads, head_dim
            128, bf16, block size 16 or 32, 512-token partitions; tables have
            room for 1024 more tokens (bench decode steps).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclass
class Workload:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    max_blocks_per_seq: int
    context_lens: np.ndarray            # int64 [num_seqs] before the decode step
    free_order: np.ndarray              # int32 permutation of 0..num_blocks-1
    seed: int
    # Sharing plan: list of (parent, child) forks applied after prefill of the
    # parents; children inherit the parent's context length.
    forks: list = field(default_factory=list)
    # Sequences that receive private tokens after forking: {seq: n_tokens}.
    extra_tokens: dict = field(default_factory=dict)
    # Sequences that are prefilled (in this order) before any fork.
    prefill_seqs: list = field(default_factory=list)
    # Sequences that get one appended token in the decode step, in order.
    step_seqs: list = field(default_factory=list)
    # Sequences decoded in the step, in order (the batch).
    decode_seqs: list = field(default_factory=list)
    partition_tokens: int = 512

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def elt_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2


def seed_for(config_index: int, repeat: int = 0) -> int:
    return config_index * 1000 + repeat


def _perm(rng: np.random.Generator, n: int) -> np.ndarray:
    return rng.permutation(n).astype(np.int32)


def tiny(repeat: int = 0) -> Workload:
    seed = seed_for(1, repeat)
    rng = np.random.default_rng(seed)
    ctx = np.array([1, 15, 16, 33], dtype=np.int64)
    return Workload(
        name="tiny", num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
        dtype=F32, num_blocks=16, max_blocks_per_seq=4, context_lens=ctx,
        free_order=_perm(rng, 16), seed=seed,
        prefill_seqs=[0, 1, 2, 3], forks=[(3, 4)],
        step_seqs=[0, 1, 2, 3], decode_seqs=[0, 1, 2, 3, 4])


def mha(repeat: int = 0, batch: int = 64) -> Workload:
    seed = seed_for(2, repeat)
    rng = np.random.default_rng(seed)
    ctx = rng.integers(1, 2048, size=batch, endpoint=True).astype(np.int64)
    nb = 16384
    return Workload(
        name="mha", num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=16,
        dtype=BF16, num_blocks=nb, max_blocks_per_seq=2048 // 16 + 32,
        context_lens=ctx, free_order=_perm(rng, nb), seed=seed,
        prefill_seqs=list(range(batch)), step_seqs=list(range(batch)),
        decode_seqs=list(range(batch)))


def gqa(repeat: int = 0, batch: int = 256) -> Workload:
    seed = seed_for(3, repeat)
    rng = np.random.default_rng(seed)
    ctx = np.rint(np.exp(rng.uniform(math.log(16), math.log(8192), size=batch))).astype(np.int64)
    bs = 16
    need = int(np.sum((ctx + bs) // bs))            # blocks incl. one appended token
    nb = int(math.ceil(1.1 * need))
    return Workload(
        name="gqa", num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=bs,
        dtype=BF16, num_blocks=nb, max_blocks_per_seq=8192 // bs + 8,
        context_lens=ctx, free_order=_perm(rng, nb), seed=seed,
        prefill_seqs=list(range(batch)), step_seqs=list(range(batch)),
        decode_seqs=list(range(batch)))


def _prefix_common(name: str, prompt_len: int, tail_max: int, seed: int,
                   prompts: int = 8, branches: int = 16) -> Workload:
    rng = np.random.default_rng(seed)
    bs = 16
    nseq = prompts * branches
    # Sequence ids: prompt i is held by branches i*branches .. i*branches+branches-1;
    # branch 0 is prefilled, the others are forked from it.
    prefill = [i * branches for i in range(prompts)]
    forks = [(i * branches, i * branches + j) for i in range(prompts) for j in range(1, branches)]
    tails = rng.integers(0, tail_max, size=nseq, endpoint=True) if tail_max > 0 else np.zeros(nseq, np.int64)
    extra = {s: int(tails[s]) for s in range(nseq) if tails[s] > 0}
    ctx = np.full(nseq, prompt_len, dtype=np.int64)
    prompt_blocks = -(-prompt_len // bs)
    private = sum(-(-(prompt_len % bs + t + 1) // bs) + 1 for t in tails)
    # + 4 blocks (64 tokens) per sequence: room for the bench's cycled decode
    # states and its end-to-end steps
    nb = int(math.ceil(1.1 * (prompts * prompt_blocks + private))) + 4 * nseq
    return Workload(
        name=name, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=bs,
        dtype=BF16, num_blocks=nb,
        max_blocks_per_seq=-(-(prompt_len + tail_max + 80) // bs),
        context_lens=ctx, free_order=_perm(rng, nb), seed=seed,
        prefill_seqs=prefill, forks=forks, extra_tokens=extra,
        step_seqs=list(range(nseq)), decode_seqs=list(range(nseq)))


def prefix(repeat: int = 0) -> Workload:
    return _prefix_common("prefix", 4000, 512, seed_for(4, repeat))


def prefix_cow(repeat: int = 0) -> Workload:
    return _prefix_common("prefix_cow", 4008, 0, seed_for(4, 100 + repeat))


def long(repeat: int = 0, block_size: int = 16, slack: float = 0.0, batch: int = 8,
         context: int = 131072) -> Workload:
    seed = seed_for(5, repeat + (0 if block_size == 16 else 50))
    rng = np.random.default_rng(seed)
    per_seq = context // block_size
    nb = batch * per_seq
    if slack > 0:
        nb = int(math.ceil(nb * (1.0 + slack)))
    ctx = np.full(batch, context, dtype=np.int64)
    return Workload(
        name=f"long_bs{block_size}", num_q_heads=64, num_kv_heads=8, head_dim=128,
        block_size=block_size, dtype=BF16, num_blocks=nb,
        max_blocks_per_seq=per_seq + 1024 // block_size, context_lens=ctx,
        free_order=_perm(rng, nb),
        seed=seed, prefill_seqs=list(range(batch)),
        step_seqs=list(range(batch)) if slack > 0 else [],
        decode_seqs=list(range(batch)), partition_tokens=512)


def random_small(seed: int, *, num_seqs: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, dtype: str, max_ctx: int,
                 min_ctx: int = 0, spare_blocks: int = 3, fixed_lens=()) -> Workload:
    """A small ragged workload for parity sweeps: uniform lengths in
    [min_ctx, max_ctx], the first ``len(fixed_lens)`` lengths set as given."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(min_ctx, max_ctx, size=num_seqs, endpoint=True).astype(np.int64)
    ctx[:len(fixed_lens)] = fixed_lens
    max_ctx = max(max_ctx, int(ctx.max()) if num_seqs else 0)
    need = int(np.sum((ctx + block_size) // block_size))
    nb = need + spare_blocks
    return Workload(
        name="random_small", num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, dtype=dtype, num_blocks=nb,
        max_blocks_per_seq=-(-(max_ctx + 1) // block_size) + 1, context_lens=ctx,
        free_order=_perm(rng, nb), seed=seed, prefill_seqs=list(range(num_seqs)),
        step_seqs=[], decode_seqs=list(range(num_seqs)))


# ---------------------------------------------------------------------------
# Value draws (torch is used only as a seeded random source and for storage).

def _torch_dtype(dtype: str):
    import torch
    return torch.float32 if dtype == F32 else torch.bfloat16


def draw_normal(shape, dtype: str, seed: int, device="cpu"):
    """N(0, 1) tensor of ``shape`` in ``dtype`` from a dedicated seeded generator."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(int(s) for s in shape), generator=g, device=device,
                    dtype=torch.float32)
    return x.to(_torch_dtype(dtype))


def draw_pools(w: Workload, device="cpu"):
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    k = draw_normal(shape, w.dtype, w.seed * 10 + 1, device)
    v = draw_normal(shape, w.dtype, w.seed * 10 + 2, device)
    return k, v


def draw_queries(w: Workload, num_seqs: int, step: int = 0, device="cpu"):
    return draw_normal((num_seqs, w.num_q_heads, w.head_dim), w.dtype,
                       w.seed * 10 + 3 + 1000 * step, device)


def draw_new_kv(w: Workload, num_tokens: int, step: int = 0, device="cpu"):
    shape = (num_tokens, w.num_kv_heads, w.head_dim)
    k = draw_normal(shape, w.dtype, w.seed * 10 + 4 + 1000 * step, device)
    v = draw_normal(shape, w.dtype, w.seed * 10 + 5 + 1000 * step, device)
    return k, v


WORKLOADS = {
    "tiny": tiny,
    "mha": mha,
    "gqa": gqa,
    "prefix": prefix,
    "prefix_cow": prefix_cow,
    "long": long,
}
