"""Paged decode attention as its definition, in float64 (test infrastructure).

Layout conventions shared with the GPU path (they are the interface, not an
implementation detail):

* ``k_pool``, ``v_pool``: ``[num_blocks, num_kv_heads, block_size, head_dim]``.
  One (physical block, KV head) tile holds ``block_size`` consecutive tokens.
* ``block_tables``: ``[num_seqs, max_blocks_per_seq]`` integers; entry
  ``[s, i]`` is the physical block that holds logical block ``i`` of
  sequence ``s``. Entries at or past ``ceil(ctx_s / block_size)`` are never read.
* ``q``: ``[num_seqs, num_q_heads, head_dim]``; query head ``h`` reads KV head
  ``h // (num_q_heads // num_kv_heads)`` (consecutive query heads share a KV
  head; the pages name grouped-query attention without fixing the map, this is
  the plainest reading).
* ``slot_mapping``: slot = physical_block * block_size + offset; a negative
  slot is padding and writes nothing.

What is computed follows two passages:

* "What is PagedAttention?" (qubittool glossary), How It Works / Map Logical
  to Physical Blocks: a block table maps each logical block index to a
  physical block ID, so one sequence's blocks need not be adjacent.
* "PagedAttention: Optimizing KV Cache in vLLM" (grasp.study), section 3
  (Making it Work: The PagedAttention Kernel): the kernel walks the blocks in
  logical order and the result is the same as attention over a contiguous
  layout. That contiguous result is what this module writes out directly.
"""

from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def gather_sequence(pool, block_table_row, context_len: int, kv_head: int) -> np.ndarray:
    """Keys (or values) of one sequence and KV head in logical token order.

    Logical token ``t`` lives in logical block ``t // block_size`` at offset
    ``t % block_size``; the block table turns the logical block into the
    physical one (qubittool glossary, How It Works). All ``context_len``
    tokens are looked up at once with that rule (array indexing, no loop).
    A negative table entry (a block released before a sliding window, never
    attended to) yields NaN rows.

    Returns float64 ``[context_len, head_dim]``.
    """
    pool = np.asarray(pool)
    block_size = pool.shape[2]
    t = np.arange(int(context_len))
    logical_block = t // block_size
    offset = t % block_size
    table = np.asarray(block_table_row, dtype=np.int64)
    physical_block = table[logical_block]
    released = physical_block < 0
    rows = pool[np.where(released, 0, physical_block), kv_head, offset, :].astype(np.float64)
    rows[released, :] = np.nan
    return rows


def attention_definition(q_vec, K, V, scale: float) -> np.ndarray:
    """softmax(scale * K q) V for one query vector, two-pass, float64.

    ``q_vec`` [D], ``K`` [n, D], ``V`` [n, D]. With n == 0 the weights are empty
    and the output is defined as zeros (no tokens to attend to).
    """
    q_vec = _f64(q_vec)
    K = _f64(K)
    V = _f64(V)
    n = K.shape[0]
    if n == 0:
        return np.zeros(V.shape[1] if V.ndim == 2 else q_vec.shape[0], dtype=np.float64)
    z = scale * (K @ q_vec)            # logits, one per token
    zmax = np.max(z)                   # pass 1: the maximum
    e = np.exp(z - zmax)               # pass 2: shifted exponentials
    p = e / np.sum(e)                  # normalised weights, sum to 1
    return p @ V


def _group(num_q_heads: int, num_kv_heads: int) -> int:
    if num_kv_heads <= 0 or num_q_heads % num_kv_heads != 0:
        raise ValueError("num_q_heads must be a positive multiple of num_kv_heads")
    return num_q_heads // num_kv_heads


def paged_decode_one(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                     seq: int, q_head: int) -> np.ndarray:
    """Decode output of one (sequence, query head): float64 [head_dim]."""
    q = np.asarray(q)
    num_q_heads = q.shape[1]
    num_kv_heads = np.asarray(k_pool).shape[1]
    kv_head = q_head // _group(num_q_heads, num_kv_heads)
    ctx = int(context_lens[seq])
    K = gather_sequence(k_pool, block_tables[seq], ctx, kv_head)
    V = gather_sequence(v_pool, block_tables[seq], ctx, kv_head)
    return attention_definition(q[seq, q_head], K, V, scale)


def paged_decode(q, k_pool, v_pool, block_tables, context_lens, scale: float) -> np.ndarray:
    """Single-query decode attention for every sequence and query head.

    Each sequence's keys and values are gathered once per KV head and serve
    every query head of that head's group (the same values
    ``paged_decode_one`` gathers per query head).

    Returns float64 ``[num_seqs, num_q_heads, head_dim]``.
    """
    q = np.asarray(q)
    num_seqs, num_q_heads, head_dim = q.shape
    num_kv_heads = np.asarray(k_pool).shape[1]
    group = _group(num_q_heads, num_kv_heads)
    out = np.zeros((num_seqs, num_q_heads, head_dim), dtype=np.float64)
    for s in range(num_seqs):
        ctx = int(context_lens[s])
        for kv_head in range(num_kv_heads):
            K = gather_sequence(k_pool, block_tables[s], ctx, kv_head)
            V = gather_sequence(v_pool, block_tables[s], ctx, kv_head)
            for h in range(kv_head * group, (kv_head + 1) * group):
                out[s, h] = attention_definition(q[s, h], K, V, scale)
    return out


def paged_decode_window(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                        window: int) -> np.ndarray:
    """Sliding-window decode: each query attends to the last ``window`` tokens
    of its sequence only (all of them when the sequence is shorter). The
    pages name sliding-window attention as a KV-cache optimisation beside
    paged attention ("PagedAttention" knowledge page, Core Facts); the window
    is the plain reading: tokens max(0, ctx - window) .. ctx - 1.

    Returns float64 ``[num_seqs, num_q_heads, head_dim]``.
    """
    if window <= 0:
        raise ValueError("window must be positive")
    q = np.asarray(q)
    num_seqs, num_q_heads, head_dim = q.shape
    num_kv_heads = np.asarray(k_pool).shape[1]
    group = _group(num_q_heads, num_kv_heads)
    out = np.zeros((num_seqs, num_q_heads, head_dim), dtype=np.float64)
    for s in range(num_seqs):
        ctx = int(context_lens[s])
        lo = max(0, ctx - window)
        for h in range(num_q_heads):
            K = gather_sequence(k_pool, block_tables[s], ctx, h // group)[lo:]
            V = gather_sequence(v_pool, block_tables[s], ctx, h // group)[lo:]
            out[s, h] = attention_definition(q[s, h], K, V, scale)
    return out


def paged_prefill(q, k_pool, v_pool, block_tables, context_lens, query_lens,
                  scale: float) -> np.ndarray:
    """Prefill (chunked prefill) attention over the paged cache, float64.

    Sequence s holds context_lens[s] tokens, of which its last query_lens[s]
    are new; their queries are rows query_start[s] .. of ``q``
    ``[total_new_tokens, num_q_heads, head_dim]`` (sequences back to back).
    New token i of sequence s sits at position p = ctx_s - qlen_s + i and
    attends to tokens 0 .. p of its sequence (causal). Prefill is the step
    that writes a request's first KV blocks before decoding ("What is
    PagedAttention?", How It Works: prefill allocates enough blocks for the
    input); the attention itself is the plain causal definition.

    Written for all of a sequence's new tokens of one query head at once:
    the logits z[i, j] = scale * q_i . k_j are kept where j <= p_i and set to
    -inf elsewhere (the causal mask), each row is normalised two-pass (its
    maximum, then exponentials and their sum), and the rows of weights
    multiply V.
    """
    q = np.asarray(q)
    total, num_q_heads, head_dim = q.shape
    num_kv_heads = np.asarray(k_pool).shape[1]
    group = _group(num_q_heads, num_kv_heads)
    out = np.zeros((total, num_q_heads, head_dim), dtype=np.float64)
    row = 0
    for s in range(len(context_lens)):
        ctx = int(context_lens[s])
        qlen = int(query_lens[s])
        if qlen > ctx:
            raise ValueError("query_lens[s] must not exceed context_lens[s]")
        if qlen == 0:
            continue
        position = np.arange(ctx - qlen, ctx)                     # of each new token
        visible = np.arange(ctx)[None, :] <= position[:, None]    # [qlen, ctx]
        for kv_head in range(num_kv_heads):
            K = gather_sequence(k_pool, block_tables[s], ctx, kv_head)
            V = gather_sequence(v_pool, block_tables[s], ctx, kv_head)
            for h in range(kv_head * group, (kv_head + 1) * group):
                Q = _f64(q[row:row + qlen, h])                    # [qlen, D]
                z = np.where(visible, scale * (Q @ K.T), -np.inf)
                zmax = np.max(z, axis=1, keepdims=True)           # pass 1: row maxima
                e = np.exp(z - zmax)                              # masked entries give 0
                p = e / np.sum(e, axis=1, keepdims=True)
                out[row:row + qlen, h] = p @ V
        row += qlen
    if row != total:
        raise ValueError("sum of query_lens must equal q.shape[0]")
    return out


def partitioned_decode_one(q, k_pool, v_pool, block_tables, context_lens, scale: float,
                           seq: int, q_head: int, partition_tokens: int) -> np.ndarray:
    """Split-context route to the same result, step by step, float64.

    The context is cut into consecutive partitions of ``partition_tokens``
    tokens. For each partition p with logits z (scaled) and values V_p:

        m_p = max z,   l_p = sum exp(z - m_p),   o_p = sum exp(z - m_p) v / l_p

    and the partitions are merged with log-sum-exp weights:

        M = max_p m_p,   w_p = l_p exp(m_p - M),   out = sum_p w_p o_p / sum_p w_p.

    The merge is an algebraic identity, so this equals ``paged_decode_one``
    up to rounding (the grasp.study lesson, section 3, states the running
    normalisation reproduces the contiguous result).
    """
    if partition_tokens <= 0:
        raise ValueError("partition_tokens must be positive")
    q = np.asarray(q)
    num_q_heads = q.shape[1]
    num_kv_heads = np.asarray(k_pool).shape[1]
    kv_head = q_head // _group(num_q_heads, num_kv_heads)
    ctx = int(context_lens[seq])
    K = gather_sequence(k_pool, block_tables[seq], ctx, kv_head)
    V = gather_sequence(v_pool, block_tables[seq], ctx, kv_head)
    qv = _f64(q[seq, q_head])
    ms, ls, os_ = [], [], []
    for start in range(0, ctx, partition_tokens):
        Kp = K[start:start + partition_tokens]
        Vp = V[start:start + partition_tokens]
        z = scale * (Kp @ qv)
        m_p = np.max(z)
        e = np.exp(z - m_p)
        l_p = np.sum(e)
        ms.append(m_p)
        ls.append(l_p)
        os_.append((e @ Vp) / l_p)
    if not ms:
        return np.zeros(qv.shape[0], dtype=np.float64)
    M = max(ms)
    w = np.array([l_p * np.exp(m_p - M) for m_p, l_p in zip(ms, ls)])
    O = np.stack(os_)
    return (w @ O) / np.sum(w)


def kv_append(k_pool, v_pool, k_new, v_new, slot_mapping) -> None:
    """Write each new token's K and V into its slot, in place.

    ``k_new``/``v_new``: ``[num_tokens, num_kv_heads, head_dim]``. Token ``t`` goes
    to physical block ``slot // block_size`` at offset ``slot % block_size`` for
    every KV head; a negative slot writes nothing. Decoding appends into the
    partly filled tail block ("What is PagedAttention?", How It Works).
    Works on any element type (bit-exact copy of the values).
    """
    block_size = k_pool.shape[2]
    num_kv_heads = k_pool.shape[1]
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        block = slot // block_size
        offset = slot % block_size
        for h in range(num_kv_heads):
            k_pool[block, h, offset, :] = k_new[t, h, :]
            v_pool[block, h, offset, :] = v_new[t, h, :]


def copy_blocks(k_pool, v_pool, src_dst_pairs) -> None:
    """Copy whole physical blocks (all heads, all slots, K and V), in place.

    This is the data movement of copy-on-write: the writer gets a private
    block holding the shared block's contents ("PagedAttention: Optimizing KV
    Cache in vLLM", section 4, step 3). Pairs are applied in order.
    """
    for pair in src_dst_pairs:
        src, dst = int(pair[0]), int(pair[1])
        k_pool[dst] = k_pool[src].copy()
        v_pool[dst] = v_pool[src].copy()
