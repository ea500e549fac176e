"""Pins of the oracle's SwitchGLU and MoE combine: closed forms on hand-built
weights and the reductions of the combine to a plain unsort and a mean."""

import math

import numpy as np

import oracle as O
from inputs import bf16_bits


def _identity_like(E, N, K, group, bits, scale=1.0):
    """Quantised weights whose dequantised value is ``scale * (n == k)``: code 1 on
    the diagonal, 0 elsewhere, step ``scale`` and bias 0 (dyadic scale)."""
    codes = np.zeros((E, N, K), np.int64)
    for n in range(min(N, K)):
        codes[:, n, n] = 1
    packed = O.pack_codes(codes.reshape(E * N, K), bits).reshape(E, N, -1)
    s = np.full((E, N, K // group), bf16_bits(np.float32(scale)), np.uint16)
    b = np.zeros((E, N, K // group), np.uint16)
    return packed, s, b


def test_switch_glu_closed_form():
    """With up = a*I, gate = c*I and down = d*I: y = d * bf16(silu(c*x) * a*x)."""
    E, H, I, group, bits = 3, 64, 64, 32, 4
    a, c, d = 0.5, 2.0, 0.25
    up = (*_identity_like(E, I, H, group, bits, a), group, bits)
    gate = (*_identity_like(E, I, H, group, bits, c), group, bits)
    down = (*_identity_like(E, H, I, group, bits, d), group, bits)
    rng = np.random.default_rng(4)
    x = bf16_bits(rng.standard_normal((5, H)).astype(np.float32))
    idx = rng.integers(0, E, size=(5, 2))
    y, h = O.switch_glu(x, idx, up, gate, down)
    xf = O.f32_from_bf16(x).astype(np.float64)
    for t in range(5):
        for k in range(2):
            for j in range(H):
                g = c * xf[t, j]
                hv = g / (1.0 + math.exp(-g)) * (a * xf[t, j])
                hb = O.f32_from_bf16(bf16_bits(np.float32(hv)))[0]
                assert h[t, k, j] == bf16_bits(np.float32(hv))[0]
                assert y[t, k, j] == d * float(hb)


def test_switch_glu_routes_each_row_to_its_expert():
    """Expert e scales by (e+1)/8: the output of row (t, k) reveals which expert ran."""
    E, H, group, bits = 4, 32, 32, 4
    ups = [_identity_like(1, H, H, group, bits, (e + 1) / 8) for e in range(E)]
    up = (np.concatenate([u[0] for u in ups]), np.concatenate([u[1] for u in ups]),
          np.concatenate([u[2] for u in ups]), group, bits)
    gate = (*_identity_like(E, H, H, group, bits, 1.0), group, bits)
    down = (*_identity_like(E, H, H, group, bits, 1.0), group, bits)
    x = bf16_bits(np.full((3, H), 1.0, np.float32))
    idx = np.array([[0, 3], [2, 1], [3, 3]])
    y, _ = O.switch_glu(x, idx, up, gate, down)
    silu1 = 1.0 / (1.0 + math.exp(-1.0))
    for t in range(3):
        for k in range(2):
            want = float(O.f32_from_bf16(bf16_bits(np.float32(silu1 * (idx[t, k] + 1) / 8)))[0])
            assert np.all(y[t, k] == want)


def test_silu_values():
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(1.0) - 0.7310585786300049) < 1e-15
    assert abs(O.silu(-1.0) + 0.2689414213699951) < 1e-15


def test_combine_reduces_to_unsort_and_mean():
    rng = np.random.default_rng(8)
    T, K, H = 6, 3, 16
    keys = rng.integers(0, 5, size=T * K)
    order, inv, _ = O.sort_by_expert(keys, 5)
    y_tok = bf16_bits(rng.standard_normal((T * K, H)).astype(np.float32))
    y_sorted = y_tok[order]
    # top_k = 1 view: score 1 and no shared expert gives back the token-order rows.
    ones = np.ones((T * K, 1), np.float32)
    out = O.moe_combine(y_sorted, inv, ones)
    assert np.array_equal(out, O.f32_from_bf16(y_tok).astype(np.float64))
    # uniform scores 1/K (exact for K = 4) give the mean over the top_k rows
    K4 = 4
    keys = rng.integers(0, 5, size=T * K4)
    order, inv, _ = O.sort_by_expert(keys, 5)
    y_tok = bf16_bits(rng.standard_normal((T * K4, H)).astype(np.float32))
    out = O.moe_combine(y_tok[order], inv, np.full((T, K4), 0.25, np.float32))
    want = O.f32_from_bf16(y_tok).astype(np.float64).reshape(T, K4, H).mean(axis=1)
    assert np.allclose(out, want, rtol=0, atol=1e-15)


def test_combine_shared_gate_closed_forms():
    rng = np.random.default_rng(9)
    T, K, H = 4, 2, 8
    y = bf16_bits(rng.standard_normal((T * K, H)).astype(np.float32))
    inv = np.arange(T * K)
    zeros = np.zeros((T, K), np.float32)
    shared = bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    x = bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wz = np.zeros(H, np.uint16)
    out = O.moe_combine(y, inv, zeros, shared, x, wz)   # sigmoid(0) = 1/2
    assert np.array_equal(out, 0.5 * O.f32_from_bf16(shared).astype(np.float64))
    # gate weight e_0 with x[:, 0] = 0 also gives 1/2; a large positive logit gives ~1
    w0 = bf16_bits(np.eye(H, dtype=np.float32)[0])
    x0 = x.copy()
    x0[:, 0] = bf16_bits(np.float32(0.0))
    assert np.array_equal(O.moe_combine(y, inv, zeros, shared, x0, w0), out)
    x0[:, 0] = bf16_bits(np.float32(60.0))
    big = O.moe_combine(y, inv, zeros, shared, x0, w0)
    assert np.allclose(big, O.f32_from_bf16(shared).astype(np.float64), rtol=1e-20, atol=1e-25)


# ------------------------------------------------------------- stock-tail combine
def _bf16_of(values):
    return bf16_bits(np.asarray(values, np.float32))


def test_stock_combine_top1_unit_score_is_the_unsort():
    """top_k = 1, score 1, no shared term: every rounding is exact, so the result is
    the expert-sorted rows put back in token order, bit for bit."""
    rng = np.random.default_rng(11)
    T, H = 6, 16
    y = _bf16_of(rng.standard_normal((T, H)))
    inv = rng.permutation(T).astype(np.uint32)
    out = O.moe_combine_stock(y, inv, np.ones((T, 1), np.float32))
    assert np.array_equal(out, y[inv.astype(np.int64)])


def test_stock_combine_equals_exact_combine_when_every_step_is_exact():
    """Small integer rows, power-of-two scores and a shared term gated by sigmoid(0) =
    1/2: every product and partial sum is a bf16 value, so the stepwise result equals
    the fp64 combine exactly."""
    rng = np.random.default_rng(12)
    T, top_k, H = 5, 4, 16
    y = _bf16_of(rng.integers(-7, 8, size=(T * top_k, H)))
    inv = rng.permutation(T * top_k).astype(np.uint32)
    scores = rng.choice(np.float32([0.25, 0.5, 1.0]), size=(T, top_k)).astype(np.float32)
    shared = _bf16_of(rng.integers(-6, 7, size=(T, H)))
    z = _bf16_of(np.zeros(T))
    got = O.moe_combine_stock(y, inv, scores, shared, z)
    # gate 1/2 in the fp64 combine: x . w_shared_gate = 0
    want = O.moe_combine(y, inv, scores, shared, _bf16_of(np.ones((T, H))), _bf16_of(np.zeros(H)))
    assert np.array_equal(got, _bf16_of(want))


def test_stock_combine_within_rounding_bound_of_exact_combine():
    """Random rows: the stepwise result differs from the fp64 combine by at most the
    roundings it performs (unit roundoff u = 2^-8 of bf16): scores and products
    (2u per term), the top_k sum (u) and the final add (u)."""
    rng = np.random.default_rng(13)
    T, top_k, H = 16, 8, 64
    y = _bf16_of(rng.standard_normal((T * top_k, H)))
    inv = rng.permutation(T * top_k).astype(np.uint32)
    p = rng.random((T, top_k)).astype(np.float32)
    scores = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    shared = _bf16_of(rng.standard_normal((T, H)))
    got = O.f32_from_bf16(O.moe_combine_stock(y, inv, scores, shared)).astype(np.float64)
    want = O.moe_combine(y, inv, scores, shared)
    yf = O.f32_from_bf16(y).astype(np.float64)[inv.astype(np.int64)].reshape(T, top_k, H)
    terms = np.abs(yf * scores.astype(np.float64)[:, :, None]).sum(axis=1)
    u = 2.0 ** -8
    bound = 3.1 * u * terms + 1.1 * u * (np.abs(want) + np.abs(O.f32_from_bf16(shared)))
    err = np.abs(got - want)
    assert np.all(err <= bound + 1e-30)
    assert err.max() > 0  # the steps do round


def test_stock_combine_gate_closed_forms():
    """Zero scores leave the gated shared term: logit 0 gives sigmoid 1/2, which halves
    bf16 values exactly; logit 30 gives a sigmoid that rounds to 1 in float32."""
    rng = np.random.default_rng(14)
    T, top_k, H = 4, 2, 16
    y = _bf16_of(rng.standard_normal((T * top_k, H)))
    inv = np.arange(T * top_k, dtype=np.uint32)
    zero = np.zeros((T, top_k), np.float32)
    shared = _bf16_of(rng.standard_normal((T, H)))
    half = O.moe_combine_stock(y, inv, zero, shared, _bf16_of(np.zeros(T)))
    assert np.array_equal(half, _bf16_of(O.f32_from_bf16(shared) / 2))
    one = O.moe_combine_stock(y, inv, zero, shared, _bf16_of(np.full(T, 30.0)))
    assert np.array_equal(one, shared)
