"""Pins for the attention oracle (CPU only).

Each test checks the oracle against something that is not the oracle: a
library routine (torch scaled_dot_product_attention in float64 over the
contiguous sequence), a closed form, or an invariant the pages state
("PagedAttention: Optimizing KV Cache in vLLM", section 3: the block-aware
walk gives the same result as a contiguous layout; "What is
PagedAttention?", How It Works: physical placement is free, only logical
order matters).
"""

import math

import numpy as np
import pytest
import torch

import oracle



def _place(contig_k, contig_v, block_size, num_blocks, rng):
    """Scatter contiguous per-sequence K/V [B][ctx, Hkv, D] into a shuffled pool.

    Built token by token with flat slot arithmetic (slot = block*bs + offset on
    a token-major view), independently of the oracle's gather loop.
    """
    B = len(contig_k)
    Hkv, D = contig_k[0].shape[1], contig_k[0].shape[2]
    max_blocks = max(1, max(-(-k.shape[0] // block_size) for k in contig_k))
    perm = rng.permutation(num_blocks)
    tables = np.full((B, max_blocks), -1, dtype=np.int64)
    flat_k = np.zeros((num_blocks * block_size, Hkv, D))
    flat_v = np.zeros((num_blocks * block_size, Hkv, D))
    nxt = 0
    for s in range(B):
        nb = -(-contig_k[s].shape[0] // block_size)
        for i in range(nb):
            tables[s, i] = perm[nxt]
            nxt += 1
        for t in range(contig_k[s].shape[0]):
            slot = tables[s, t // block_size] * block_size + t % block_size
            flat_k[slot] = contig_k[s][t]
            flat_v[slot] = contig_v[s][t]
    # token-major [NB*bs, H, D] -> [NB, H, bs, D]
    k_pool = flat_k.reshape(num_blocks, block_size, Hkv, D).transpose(0, 2, 1, 3).copy()
    v_pool = flat_v.reshape(num_blocks, block_size, Hkv, D).transpose(0, 2, 1, 3).copy()
    return k_pool, v_pool, tables


def _sdpa_reference(q, contig_k, contig_v, scale):
    """torch SDPA (float64, CPU) per sequence over the contiguous K/V."""
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D))
    for s in range(B):
        K = torch.from_numpy(contig_k[s])  # [ctx, Hkv, D]
        V = torch.from_numpy(contig_v[s])
        ctx, Hkv, _ = K.shape
        if ctx == 0:
            continue
        g = Hq // Hkv
        Kh = K.permute(1, 0, 2).repeat_interleave(g, dim=0)  # [Hq, ctx, D]
        Vh = V.permute(1, 0, 2).repeat_interleave(g, dim=0)
        qh = torch.from_numpy(q[s]).unsqueeze(1)            # [Hq, 1, D]
        o = torch.nn.functional.scaled_dot_product_attention(qh, Kh, Vh, scale=scale)
        out[s] = o.squeeze(1).numpy()
    return out


@pytest.mark.parametrize("Hq,Hkv,D,bs,lens", [
    (2, 2, 64, 16, [1, 15, 16, 33]),
    (4, 2, 32, 16, [5, 0, 47, 16, 17]),
    (8, 1, 16, 32, [31, 32, 33, 100]),
    (6, 3, 8, 8, [1, 2, 9, 64]),
])
def test_matches_sdpa_float64(Hq, Hkv, D, bs, lens):
    rng = np.random.default_rng(123 + Hq + bs)
    contig_k = [rng.standard_normal((n, Hkv, D)) for n in lens]
    contig_v = [rng.standard_normal((n, Hkv, D)) for n in lens]
    nb = sum(-(-n // bs) for n in lens) + 5
    k_pool, v_pool, tables = _place(contig_k, contig_v, bs, nb, rng)
    q = rng.standard_normal((len(lens), Hq, D))
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_decode(q, k_pool, v_pool, tables, np.array(lens), scale)
    want = _sdpa_reference(q, contig_k, contig_v, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_single_token_returns_its_value():
    rng = np.random.default_rng(1)
    k_pool = rng.standard_normal((4, 1, 16, 8))
    v_pool = rng.standard_normal((4, 1, 16, 8))
    tables = np.array([[2, 0]])
    q = rng.standard_normal((1, 1, 8)) * 50.0
    out = oracle.paged_decode(q, k_pool, v_pool, tables, np.array([1]), 0.3)
    assert np.array_equal(out[0, 0], v_pool[2, 0, 0])


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(2)
    bs, ctx = 16, 37
    k_pool = np.zeros((5, 1, bs, 4))
    k_pool[:, 0, :, :] = rng.standard_normal(4)  # every slot holds the same key
    v_pool = rng.standard_normal((5, 1, bs, 4))
    tables = np.array([[4, 1, 3]])
    q = rng.standard_normal((1, 1, 4))
    out = oracle.paged_decode(q, k_pool, v_pool, tables, np.array([ctx]), 0.7)
    vals = np.concatenate([v_pool[4, 0], v_pool[1, 0], v_pool[3, 0][:ctx - 32]])
    np.testing.assert_allclose(out[0, 0], vals.mean(axis=0), rtol=0, atol=1e-14)


def test_two_token_worked_example():
    # logits 0 and ln 3 -> weights 1/4 and 3/4 (closed form)
    k_pool = np.zeros((2, 1, 2, 2))
    v_pool = np.zeros((2, 1, 2, 2))
    k_pool[1, 0, 0] = [0.0, 0.0]
    k_pool[1, 0, 1] = [math.log(3.0), 0.0]
    v_pool[1, 0, 0] = [1.0, -2.0]
    v_pool[1, 0, 1] = [5.0, 2.0]
    q = np.array([[[1.0, 7.0]]])
    out = oracle.paged_decode(q, k_pool, v_pool, np.array([[1]]), np.array([2]), 1.0)
    np.testing.assert_allclose(out[0, 0], [0.25 * 1 + 0.75 * 5, 0.25 * -2 + 0.75 * 2], atol=1e-15)


def test_zero_context_gives_zeros():
    k_pool = np.ones((2, 1, 4, 3))
    out = oracle.paged_decode(np.ones((1, 1, 3)), k_pool, k_pool, np.array([[0]]), np.array([0]), 1.0)
    assert np.array_equal(out, np.zeros((1, 1, 3)))


def test_physical_placement_is_irrelevant():
    rng = np.random.default_rng(3)
    bs, nb, Hkv, D = 16, 12, 2, 8
    k_pool = rng.standard_normal((nb, Hkv, bs, D))
    v_pool = rng.standard_normal((nb, Hkv, bs, D))
    tables = np.array([[3, 7, 1, -1], [0, 11, 5, 9]])
    lens = np.array([40, 64])
    q = rng.standard_normal((2, 4, D))
    base = oracle.paged_decode(q, k_pool, v_pool, tables, lens, 0.25)
    perm = rng.permutation(nb)          # block b moves to perm[b]
    k2 = np.empty_like(k_pool)
    v2 = np.empty_like(v_pool)
    k2[perm] = k_pool
    v2[perm] = v_pool
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    moved = oracle.paged_decode(q, k2, v2, t2, lens, 0.25)
    assert np.array_equal(base, moved)


def test_common_logit_shift_is_invisible():
    rng = np.random.default_rng(4)
    k_pool = rng.standard_normal((3, 1, 8, 6))
    v_pool = rng.standard_normal((3, 1, 8, 6))
    q = rng.standard_normal((1, 1, 6))
    tables = np.array([[2, 0, 1]])
    base = oracle.paged_decode(q, k_pool, v_pool, tables, np.array([20]), 0.5)
    shifted = k_pool + 3.0 * q[0, 0] / np.dot(q[0, 0], q[0, 0])   # every logit +1.5
    out = oracle.paged_decode(q, shifted, v_pool, tables, np.array([20]), 0.5)
    np.testing.assert_allclose(out, base, rtol=0, atol=1e-13)


def test_large_logits_stay_finite_and_pick_the_top_key():
    rng = np.random.default_rng(5)
    k_pool = rng.standard_normal((2, 1, 16, 4))
    v_pool = rng.standard_normal((2, 1, 16, 4))
    q = np.array([[[1000.0, 0.0, 0.0, 0.0]]])
    k_pool[1, 0, 9, 0] = 10.0          # logit 1e4, the next best is < 4e3
    out = oracle.paged_decode(q, k_pool, v_pool, np.array([[0, 1]]), np.array([32]), 1.0)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out[0, 0], v_pool[1, 0, 9], atol=1e-12)


def test_gqa_head_map_is_consecutive_groups():
    # 4 query heads over 2 KV heads: heads {0,1} read KV head 0, {2,3} read KV head 1.
    D, bs = 4, 4
    k_pool = np.zeros((1, 2, bs, D))
    v_pool = np.zeros((1, 2, bs, D))
    v_pool[0, 0] = 1.0
    v_pool[0, 1] = -1.0
    q = np.ones((1, 4, D))
    out = oracle.paged_decode(q, k_pool, v_pool, np.array([[0]]), np.array([3]), 1.0)
    assert np.array_equal(out[0, :, 0], [1.0, 1.0, -1.0, -1.0])


@pytest.mark.parametrize("part", [1, 3, 16, 17, 50, 64, 200])
def test_partitioned_merge_equals_definition(part):
    rng = np.random.default_rng(6)
    bs, D = 16, 8
    k_pool = rng.standard_normal((6, 2, bs, D)) * 3
    v_pool = rng.standard_normal((6, 2, bs, D))
    q = rng.standard_normal((1, 4, D))
    tables = np.array([[5, 2, 0, 3]])
    lens = np.array([50])
    for h in range(4):
        want = oracle.paged_decode_one(q, k_pool, v_pool, tables, lens, 0.4, 0, h)
        got = oracle.partitioned_decode_one(q, k_pool, v_pool, tables, lens, 0.4, 0, h, part)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_kv_append_against_flat_slot_view():
    rng = np.random.default_rng(7)
    nb, H, bs, D = 5, 3, 16, 4
    k_pool = rng.standard_normal((nb, H, bs, D))
    v_pool = rng.standard_normal((nb, H, bs, D))
    k_new = rng.standard_normal((4, H, D))
    v_new = rng.standard_normal((4, H, D))
    slots = np.array([37, -1, 0, 79])
    ek = k_pool.transpose(0, 2, 1, 3).reshape(nb * bs, H, D).copy()
    ev = v_pool.transpose(0, 2, 1, 3).reshape(nb * bs, H, D).copy()
    for t, s in enumerate(slots):
        if s >= 0:
            ek[s] = k_new[t]
            ev[s] = v_new[t]
    oracle.kv_append(k_pool, v_pool, k_new, v_new, slots)
    assert np.array_equal(k_pool.transpose(0, 2, 1, 3).reshape(nb * bs, H, D), ek)
    assert np.array_equal(v_pool.transpose(0, 2, 1, 3).reshape(nb * bs, H, D), ev)
    # worked example: slot 37 with block size 16 is block 2, offset 5
    assert np.array_equal(k_pool[2, :, 5, :], k_new[0])


def test_copy_blocks_hand_example():
    k_pool = np.arange(4 * 2 * 2 * 2, dtype=np.float64).reshape(4, 2, 2, 2)
    v_pool = -k_pool
    k0, v0 = k_pool.copy(), v_pool.copy()
    oracle.copy_blocks(k_pool, v_pool, [(1, 3), (0, 2)])
    assert np.array_equal(k_pool[3], k0[1]) and np.array_equal(v_pool[3], v0[1])
    assert np.array_equal(k_pool[2], k0[0]) and np.array_equal(v_pool[2], v0[0])
    assert np.array_equal(k_pool[:2], k0[:2]) and np.array_equal(v_pool[:2], v0[:2])


def test_window_covering_the_context_is_plain_decode():
    rng = np.random.default_rng(8)
    k_pool = rng.standard_normal((6, 2, 16, 8))
    v_pool = rng.standard_normal((6, 2, 16, 8))
    q = rng.standard_normal((2, 4, 8))
    tables = np.array([[5, 1, 3, 0], [2, 4, -1, -1]])
    lens = np.array([50, 20])
    full = oracle.paged_decode(q, k_pool, v_pool, tables, lens, 0.3)
    for w in (50, 64, 10_000):
        assert np.array_equal(oracle.paged_decode_window(q, k_pool, v_pool, tables, lens, 0.3, w)[0], full[0])


def test_window_of_one_returns_the_last_value():
    rng = np.random.default_rng(9)
    k_pool = rng.standard_normal((4, 1, 16, 8))
    v_pool = rng.standard_normal((4, 1, 16, 8))
    q = rng.standard_normal((1, 2, 8)) * 20
    tables = np.array([[3, 0, 2]])
    out = oracle.paged_decode_window(q, k_pool, v_pool, tables, np.array([37]), 0.2, 1)
    assert np.array_equal(out[0, 0], v_pool[2, 0, 4]) and np.array_equal(out[0, 1], v_pool[2, 0, 4])


@pytest.mark.parametrize("window", [1, 5, 16, 17, 33, 100])
def test_window_matches_sdpa_on_the_slice(window):
    rng = np.random.default_rng(10 + window)
    lens = [40, 3, 64, 90]
    contig_k = [rng.standard_normal((n, 2, 16)) for n in lens]
    contig_v = [rng.standard_normal((n, 2, 16)) for n in lens]
    k_pool, v_pool, tables = _place(contig_k, contig_v, 16, 30, rng)
    q = rng.standard_normal((4, 4, 16))
    got = oracle.paged_decode_window(q, k_pool, v_pool, tables, np.array(lens), 0.25, window)
    sliced_k = [k[max(0, len(k) - window):] for k in contig_k]
    sliced_v = [v[max(0, len(v) - window):] for v in contig_v]
    want = _sdpa_reference(q, sliced_k, sliced_v, 0.25)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    # released blocks before the window are never touched
    t2 = tables.copy()
    for s, n in enumerate(lens):
        t2[s, :max(0, n - window) // 16] = -1
    assert np.array_equal(oracle.paged_decode_window(q, k_pool, v_pool, t2, np.array(lens), 0.25, window), got)


def test_prefill_single_new_token_is_decode():
    rng = np.random.default_rng(12)
    k_pool = rng.standard_normal((8, 2, 16, 8))
    v_pool = rng.standard_normal((8, 2, 16, 8))
    tables = np.array([[1, 5, 2], [7, 0, -1]])
    lens = np.array([40, 17])
    q = rng.standard_normal((2, 4, 8))
    got = oracle.paged_prefill(q, k_pool, v_pool, tables, lens, [1, 1], 0.3)
    want = oracle.paged_decode(q, k_pool, v_pool, tables, lens, 0.3)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("prior,qlen", [(0, 7), (0, 33), (21, 12), (50, 1)])
def test_prefill_matches_sdpa_with_causal_mask(prior, qlen):
    rng = np.random.default_rng(13 + prior + qlen)
    ctx = prior + qlen
    contig_k = [rng.standard_normal((ctx, 2, 16))]
    contig_v = [rng.standard_normal((ctx, 2, 16))]
    k_pool, v_pool, tables = _place(contig_k, contig_v, 16, 12, rng)
    q = rng.standard_normal((qlen, 4, 16))
    got = oracle.paged_prefill(q, k_pool, v_pool, tables, [ctx], [qlen], 0.25)
    # SDPA over the contiguous sequence with an explicit causal mask
    K = torch.from_numpy(contig_k[0]).permute(1, 0, 2).repeat_interleave(2, dim=0)   # [Hq, ctx, D]
    V = torch.from_numpy(contig_v[0]).permute(1, 0, 2).repeat_interleave(2, dim=0)
    Q = torch.from_numpy(q).permute(1, 0, 2)                                          # [Hq, qlen, D]
    pos = torch.arange(prior, ctx).unsqueeze(1)
    mask = torch.arange(ctx).unsqueeze(0) <= pos                                      # [qlen, ctx]
    want = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=0.25)
    np.testing.assert_allclose(got, want.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    if prior == 0:
        causal = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=0.25)
        np.testing.assert_allclose(got, causal.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
