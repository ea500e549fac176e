"""Pins of the oracle's qmm and gather_qmm: exact rational brute force on tiny
shapes, and the selection identities of nuvec-core's gather_qmm_selects_batches."""

from fractions import Fraction

import numpy as np

import oracle as O
from inputs import bf16_bits, random_qweight


def _dyadic_weight(rng, E, N, K, group, bits):
    """Codes plus dyadic bf16 scales/biases, and the exact rational dequantised
    matrix built without the oracle (q*s + b over Fractions)."""
    codes = rng.integers(0, 1 << bits, size=(E, N, K))
    sq = rng.integers(-64, 64, size=(E, N, K // group))
    sq[sq == 0] = 1
    bq = rng.integers(-64, 64, size=(E, N, K // group))
    s_val, b_val = sq / 1024.0, bq / 32.0
    s = bf16_bits(s_val.astype(np.float32))
    b = bf16_bits(b_val.astype(np.float32))
    exact = [[[Fraction(int(codes[e, n, k])) * Fraction(int(sq[e, n, k // group]), 1024)
               + Fraction(int(bq[e, n, k // group]), 32) for k in range(K)]
              for n in range(N)] for e in range(E)]
    packed = O.pack_codes(codes.reshape(E * N, K), bits).reshape(E, N, -1)
    return packed, s, b, exact


def _exact_dot(xrow, wrow):
    terms = [Fraction(float(a)) * wk for a, wk in zip(xrow, wrow)]
    return sum(terms, Fraction(0)), sum((abs(t) for t in terms), Fraction(0))


def test_qmm_matches_exact_rational_brute_force():
    rng = np.random.default_rng(0x52)
    # the (bits, group) pairs of nuvec-core's quantized_matmul_equals_the_dequantized_product
    for bits, group in [(4, 64), (3, 32), (8, 128), (2, 32), (6, 64), (5, 32), (1, 64),
                        (4, 32), (8, 64), (4, 128)]:
        N, K, M = 3, 128, 2
        packed, s, b, exact = _dyadic_weight(rng, 1, N, K, group, bits)
        x = bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        xf = O.f32_from_bf16(x)
        got = O.qmm(x, packed[0], s[0], b[0], group, bits)
        for m in range(M):
            for n in range(N):
                val, mag = _exact_dot(xf[m], exact[0][n])
                assert abs(got[m, n] - float(val)) <= 1e-12 * float(mag) + 1e-300


def test_gather_qmm_matches_exact_rational_brute_force():
    rng = np.random.default_rng(0x71)
    E, N, K, M, group, bits = 3, 4, 64, 2, 32, 4
    packed, s, b, exact = _dyadic_weight(rng, E, N, K, group, bits)
    x = bf16_bits(rng.standard_normal((4, M, K)).astype(np.float32))
    xf = O.f32_from_bf16(x)
    lhs, rhs = [3, 0, 2], [1, 2, 0]
    got = O.gather_qmm(x, packed, s, b, group, bits, lhs, rhs)
    assert got.shape == (3, M, N)
    for j, (l, r) in enumerate(zip(lhs, rhs)):
        for m in range(M):
            for n in range(N):
                val, mag = _exact_dot(xf[l, m], exact[r][n])
                assert abs(got[j, m, n] - float(val)) <= 1e-12 * float(mag) + 1e-300


def test_gather_qmm_selects_batches_and_default_indices():
    """gather_qmm_selects_batches: batch j equals quantized_matmul of the selected
    x batch and weight batch; default indices broadcast x's batch."""
    rng = np.random.default_rng(0x71)
    E, N, K, group, bits = 3, 8, 64, 32, 4
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = bf16_bits(rng.random((4, 2, K)).astype(np.float32) / 4)
    got = O.gather_qmm(x, w, s, b, group, bits, [3, 0, 2], [1, 2, 0])
    for j, (l, r) in enumerate(zip([3, 0, 2], [1, 2, 0])):
        assert np.array_equal(got[j], O.qmm(x[l], w[r], s[r], b[r], group, bits))
    x1 = x[:1, :1]
    allb = O.gather_qmm(x1, w, s, b, group, bits)
    assert allb.shape == (3, 1, N)
    for e in range(E):
        assert np.array_equal(allb[e], O.qmm(x1[0], w[e], s[e], b[e], group, bits))
    # rhs only: x broadcast per token over its experts (decode layout, M = 1).
    rhs = np.array([5 % E, 1, 2, 0, 1, 1])
    xt = x[:3, :1]
    got = O.gather_qmm(xt, w, s, b, group, bits, None, rhs)
    for j in range(6):
        assert np.array_equal(got[j], O.qmm(xt[j // 2], w[rhs[j]], s[rhs[j]], b[rhs[j]], group, bits))


def test_gather_qmm_sorted_and_unsorted_indices_agree_bitwise():
    rng = np.random.default_rng(9)
    E, N, K, group, bits = 8, 16, 128, 64, 4
    w, s, b = random_qweight(rng, E, N, K, group, bits)
    x = bf16_bits(rng.standard_normal((5, 1, K)).astype(np.float32))
    lhs = np.repeat(np.arange(5), 2)
    rhs = rng.integers(0, E, size=10)
    perm = np.argsort(rhs, kind="stable")
    unsorted = O.gather_qmm(x, w, s, b, group, bits, lhs, rhs)
    sorted_ = O.gather_qmm(x, w, s, b, group, bits, lhs[perm], rhs[perm])
    assert np.array_equal(sorted_, unsorted[perm])


# ------------------------------------------------------------------ gather_mm
def test_gather_mm_matches_exact_rational_brute_force():
    """Unquantized gather_mm against exact rational dot products of the bf16 values."""
    rng = np.random.default_rng(0x91)
    E, N, K, M = 3, 5, 48, 2
    w = bf16_bits(rng.standard_normal((E, N, K)).astype(np.float32))
    x = bf16_bits(rng.standard_normal((4, M, K)).astype(np.float32))
    wf, xf = O.f32_from_bf16(w), O.f32_from_bf16(x)
    lhs, rhs = [3, 0, 2, 0], [1, 2, 0, 1]
    got = O.gather_mm(x, w, lhs, rhs)
    assert got.shape == (4, M, N)
    for j, (l, r) in enumerate(zip(lhs, rhs)):
        for m in range(M):
            for n in range(N):
                val, mag = _exact_dot(xf[l, m], [Fraction(float(v)) for v in wf[r, n]])
                assert abs(got[j, m, n] - float(val)) <= 1e-12 * float(mag) + 1e-300


def test_gather_mm_equals_gather_qmm_on_exactly_dequantised_weights():
    """With scale 1/4 and bias -2 every dequantised weight q/4 - 2 is a bf16 value, so
    gather_mm over those bf16 weights and gather_qmm over the codes agree exactly
    (index defaults and broadcast of x over the weights included)."""
    rng = np.random.default_rng(0x92)
    E, N, K, M, group, bits = 4, 6, 64, 3, 32, 4
    codes = rng.integers(0, 16, size=(E, N, K))
    packed = O.pack_codes(codes.reshape(E * N, K), bits).reshape(E, N, -1)
    s = bf16_bits(np.full((E, N, K // group), 0.25, np.float32))
    b = bf16_bits(np.full((E, N, K // group), -2.0, np.float32))
    w = bf16_bits((codes * 0.25 - 2.0).astype(np.float32))
    x = bf16_bits(rng.standard_normal((2, M, K)).astype(np.float32))
    rhs = [3, 1, 1, 0, 2]
    assert np.array_equal(O.gather_mm(x, w, None, rhs), O.gather_qmm(x, packed, s, b, group, bits, None, rhs))
    assert np.array_equal(O.gather_mm(x[:1], w), O.gather_qmm(x[:1], packed, s, b, group, bits))
