"""Pins of the oracle's bf16, packing, quantisation and dequantisation against what
the pages and arithmetic fix (CPU only)."""

import json
import os

import numpy as np
import pytest

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_round_to_nearest_even_hand_patterns():
    f = np.array([1.0, -2.0, 0.0, 3.75, -0.25], np.float32)
    assert list(O.bf16_from_f32(f)) == [0x3F80, 0xC000, 0x0000, 0x4070, 0xBE80]
    # Exact ties go to the even neighbour; anything above a tie rounds up.
    bits = np.array([0x3F808000, 0x3F818000, 0x3F808001, 0x3F807FFF], np.uint32)
    assert list(O.bf16_from_f32(bits.view(np.float32))) == [0x3F80, 0x3F82, 0x3F81, 0x3F80]
    # Overflow past the largest bf16 rounds to infinity; NaN stays NaN.
    big = np.array([0x7F7FFFFF], np.uint32).view(np.float32)
    assert O.bf16_from_f32(big)[0] == 0x7F80
    nan = O.bf16_from_f32(np.array([np.nan], np.float32))[0]
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F) != 0
    # bf16 -> f32 is exact: it is the top half of the f32 pattern.
    assert O.f32_from_bf16(np.array([0x3F80, 0x4070], np.uint16)).tolist() == [1.0, 3.75]


def test_bf16_from_f64_rounds_once():
    """fp64 -> bf16 is one round-to-nearest-even step (the SwitchGLU's h is rounded
    to bf16 once).  Hand patterns where rounding through float32 first would differ,
    then exact-rational nearest-even checks on random values."""
    from fractions import Fraction
    v = np.array([1 + 2.0**-8 + 2.0**-30, 1 + 2.0**-8, 1 + 3 * 2.0**-8,
                  -(1 + 2.0**-8 + 2.0**-40), 0.0, 3.75], np.float64)
    assert [int(b) for b in O.bf16_from_f64(v)] == [0x3F81, 0x3F80, 0x3F82, 0xBF81, 0x0000,
                                                      0x4070]
    rng = np.random.default_rng(11)
    vals = rng.standard_normal(400) * np.exp2(rng.integers(-60, 60, 400))
    got = O.bf16_from_f64(vals)

    def val(bits):
        return Fraction(float(O.f32_from_bf16(np.array([bits], np.uint16))[0]))

    for x, b in zip(vals, got):
        b = int(b)
        fx, here = Fraction(float(x)), val(b)
        for nb in (b - 1, b + 1):  # neighbours with the same sign, magnitude +- 1 ulp
            if (nb & 0x7FFF) == 0x7F80 or (nb & 0x8000) != (b & 0x8000):
                continue
            d0, d1 = abs(fx - here), abs(fx - val(nb))
            assert d0 < d1 or (d0 == d1 and (b & 1) == 0), (x, hex(b), hex(nb))


def test_pack_layout_hand_words():
    assert O.pack_codes(np.arange(8)[None], 4)[0, 0] == 0x76543210
    assert O.pack_codes(np.array([[1, 2, 3, 4]]), 8)[0, 0] == 0x04030201
    assert O.pack_codes(np.array([[15, 0, 0, 0, 0, 0, 0, 1]]), 4)[0, 0] == 0x1000000F
    rng = np.random.default_rng(3)
    for bits in O.CODE_BITS:
        c = rng.integers(0, 1 << bits, size=(3, 64))
        assert np.array_equal(O.unpack_codes(O.pack_codes(c, bits), bits), c)


def _one_code(n, j, v):
    c = np.zeros((1, n), np.int64)
    c[0, j] = v
    return c


def test_pack_bit_stream_hand_words():
    """Codes form one least-significant-bit-first stream per row (code j at stream bits
    [j*bits, (j+1)*bits)); [P3] fixes the packed row at cols*bits/32 words for every
    width, so 3-, 5- and 6-bit codes straddle words.  Words worked out by hand."""
    # 1 bit: codes 0 and 31 set
    c = np.zeros((1, 32), np.int64)
    c[0, 0] = c[0, 31] = 1
    assert [int(v) for v in O.pack_codes(c, 1)[0]] == [0x80000001]
    # 2 bits: 0,1,2,3 repeated -> byte 0b11100100
    assert [int(v) for v in O.pack_codes(np.arange(16)[None] % 4, 2)[0]] == [0xE4E4E4E4]
    # 3 bits: code 10 = 0b111 sits at stream bits 30..32
    assert [int(v) for v in O.pack_codes(_one_code(32, 10, 7), 3)[0]] == [0xC0000000, 0x1, 0]
    # 5 bits: code 6 = 0b10101 at stream bits 30..34
    assert [int(v) for v in O.pack_codes(_one_code(32, 6, 21), 5)[0]] == [0x40000000, 0x5, 0, 0, 0]
    # 6 bits: code 5 = 0b110011 at stream bits 30..35
    assert [int(v) for v in O.pack_codes(_one_code(32, 5, 51), 6)[0]] == \
        [0xC0000000, 0xC, 0, 0, 0, 0]
    for bits in (3, 5, 6):
        assert O.pack_codes(np.zeros((2, 64), np.int64), bits).shape == (2, 2 * bits)


def test_seven_bits_is_rejected():
    """[P3] rejected_arguments: quantize(64, 7) fails."""
    with pytest.raises(AssertionError):
        O.quantize(np.zeros((1, 64), np.float32), 64, 7)


def test_quantize_hand_example():
    g = json.load(open(os.path.join(GOLD, "quantize_hand_example.json")))
    w = ((np.arange(32) % 16) * 0.25).astype(np.float32)[None]
    packed, s, b = O.quantize(w, g["group"], g["bits"])
    assert [int(v) for v in packed[0]] == [int(h, 16) for h in g["words"]]
    assert s[0, 0] == int(g["scale_bf16"], 16) and b[0, 0] == int(g["bias_bf16"], 16)
    assert np.array_equal(O.dequantize(packed, s, b, 32, 4), w)


@pytest.mark.parametrize("bits", O.CODE_BITS)
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dist", ["uniform", "normal"])
def test_round_trip_error_is_about_half_a_step(bits, group, dist):
    """nuvec-core quantized.rs round_trip_error_is_about_half_a_step: every error
    within one step (x1.0001), the mean error within half a step (float32 scales,
    data U[0, 0.25) as in its ``random`` helper; also N(0,1))."""
    rng = np.random.default_rng(0x51 + bits + group)
    shape = (3, 2 * group)
    w = (rng.random(shape) / 4 if dist == "uniform" else rng.standard_normal(shape)).astype(np.float32)
    packed, s, b = O.quantize(w, group, bits, scale_dtype="f32")
    assert packed.dtype == np.uint32 and packed.shape == (3, 2 * group * bits // 32)
    assert s.shape == (3, 2)
    back = O.dequantize(packed, s, b, group, bits).astype(np.float64)
    step = np.repeat(np.abs(s.astype(np.float64)), group, axis=1)
    err = np.abs(back - w)
    assert np.all(err <= step * 1.0001)
    assert err.sum() <= step.sum() / 2


@pytest.mark.parametrize("bits", O.CODE_BITS)
def test_quantize_constant_negative_and_zero_spanning_groups(bits):
    """nuvec-core quantized.rs quantize_snaps_zero_and_handles_constant_and_one_signed_groups."""
    v = [0.75] * 32 + [-1.0 - i / 8 for i in range(32)] + [i / 31 - 0.25 for i in range(32)]
    w = np.array(v, np.float32).reshape(3, 32)
    packed, s, b = O.quantize(w, 32, bits, scale_dtype="f32")
    back = O.dequantize(packed, s, b, 32, bits)
    assert np.all(np.abs(back[0] - 0.75) < 1e-6)
    # all-negative group stays within one step
    assert np.all(np.abs(back[1] - w[1]) <= abs(s[1, 0]) * 1.0001)
    # zero is exactly representable in a group that spans it: some code in [0, 2^bits)
    # restores it to within 1e-7
    q = np.arange(1 << bits, dtype=np.float64)
    assert np.min(np.abs(q * s[2, 0] + b[2, 0])) < 1e-7


def test_quantize_codes_in_range_and_bf16_storage_close_to_f32():
    rng = np.random.default_rng(7)
    w = rng.standard_normal((16, 256)).astype(np.float32)
    for bits in O.CODE_BITS:
        p32, s32, b32 = O.quantize(w, 64, bits, "f32")
        p16, s16, b16 = O.quantize(w, 64, bits, "bf16")
        c = O.unpack_codes(p16, bits)
        assert c.min() >= 0 and c.max() <= (1 << bits) - 1
        back = O.dequantize(p16, s16, b16, 64, bits)
        step = np.repeat(np.abs(O.f32_from_bf16(s16)), 64, axis=1)
        # bf16 rounding of the step adds at most n * 2^-9 steps at the far end.
        n = (1 << bits) - 1
        assert np.all(np.abs(back - w) <= step * (1.0001 + n * 2.0 ** -8))


def test_dequantize_dyadic_closed_form():
    """q*s + b with dyadic s and b is exact: compare with integer arithmetic."""
    rng = np.random.default_rng(11)
    for bits in O.CODE_BITS:
        codes = rng.integers(0, 1 << bits, size=(5, 128))
        packed = O.pack_codes(codes, bits)
        sq = rng.integers(1, 64, size=(5, 2))          # s = sq / 256
        bq = rng.integers(-64, 64, size=(5, 2))        # b = bq / 16
        s = (sq / 256).astype(np.float32)
        b = (bq / 16).astype(np.float32)
        got = O.dequantize(packed, O.bf16_from_f32(s), O.bf16_from_f32(b), 64, bits)
        want = (codes * np.repeat(sq, 64, axis=1) + 16 * np.repeat(bq, 64, axis=1)) / 256.0
        assert np.array_equal(got.astype(np.float64), want)


def test_quantize_dequantize_batched_leading_dims():
    rng = np.random.default_rng(5)
    w = rng.standard_normal((6, 128)).astype(np.float32)
    p, s, b = O.quantize(w, 64, 4)
    d = O.dequantize(p.reshape(2, 3, -1), s.reshape(2, 3, -1), b.reshape(2, 3, -1), 64, 4)
    assert np.array_equal(d.reshape(6, 128), O.dequantize(p, s, b, 64, 4))
