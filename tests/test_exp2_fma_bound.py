"""The FMA-pipe 2^x of the tcgen05 prefill kernel (exp2_fma_pair in
csrc/tc_prefill_kernel.cuh), evaluated step by step in float32 with the
coefficients read from the header: round-to-integer by the 1.5 * 2^23
shift, cubic for 2^f on [-1/2, 1/2], exponent added as the shifted bits of
t. Its relative error must stay far below bf16's 2^-9 rounding of P."""

import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), "..", "paged_kv_cache_336_b200", "csrc",
                      "tc_prefill_kernel.cuh")


def _coefficients():
    src = open(HEADER).read()
    body = src[src.index("exp2_fma_pair"):]
    body = body[:body.index("\n}\n")]
    c3, c2 = re.search(r"f2_pack\(([0-9.]+)f, [0-9.]+f\), f, f2_pack\(([0-9.]+)f", body).groups()
    c1 = re.search(r"f2_fma\(p, f, f2_pack\(([0-9.]+)f", body).group(1)
    return np.float32(c3), np.float32(c2), np.float32(c1)


def _exp2_fma(x):
    c3, c2, c1 = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def test_relative_error_bound_over_the_used_range():
    x = np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32)
    rel = np.abs(_exp2_fma(x) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.5e-4
    assert rel.max() < 2.0 ** -9 / 10


def test_integers_are_exact_and_clamp_is_tiny():
    n = np.arange(-125, 9, dtype=np.float32)
    assert np.array_equal(_exp2_fma(n), np.exp2(n.astype(np.float64)))
    assert _exp2_fma(np.array([-300.0, -126.0], np.float32)).max() == 2.0 ** -125
