"""Pins of the oracle's scalar formats: E2M1 codes, E4M3 scales, bf16 rounding.

The pages name the formats (E2M1 element codes with an FP8 E4M3 scale per 16
elements: "Mix-Quant：面向智能体LLM的量化预填充与精确解码", section NVFP4 微缩放量化;
r9-hu digest, section Method, item 1) and "RTN" rounding; they print no grid.
The grids are fixed here from the formats' bit fields (a different derivation
from the oracle's tables), and rounding is checked exhaustively against a
brute-force nearest-value search written separately (tests/pins).
"""
import ctypes
import math
import random
from fractions import Fraction

import numpy as np
import pytest


def _e2m1_from_bits(c):
    s, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = 0.5 * m if e == 0 else (1 + 0.5 * m) * 2.0 ** (e - 1)
    return -mag if s else mag


def _e4m3_from_bits(c):
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    if e == 15 and m == 7:
        return math.nan
    mag = (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_e2m1_decode_matches_bit_fields(oracle_mod):
    for c in range(16):
        got = oracle_mod.e2m1_decode(c)
        want = _e2m1_from_bits(c)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), c


def test_e2m1_grid_is_the_eight_values(oracle_mod):
    mags = sorted({abs(oracle_mod.e2m1_decode(c)) for c in range(16)})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_decode_matches_bit_fields(oracle_mod):
    for c in range(256):
        got, want = oracle_mod.e4m3_decode(c), _e4m3_from_bits(c)
        if math.isnan(want):
            assert math.isnan(got), c
        else:
            assert got == want, c


def test_e4m3_landmarks(oracle_mod):
    assert oracle_mod.e4m3_decode(0x7E) == 448.0           # largest finite
    assert oracle_mod.e4m3_decode(0x01) == 2.0 ** -9       # smallest subnormal
    assert oracle_mod.e4m3_decode(0x08) == 2.0 ** -6       # smallest normal
    assert math.isnan(oracle_mod.e4m3_decode(0x7F))
    vals = [oracle_mod.e4m3_decode(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))       # codes order like values


@pytest.mark.parametrize("codes", [range(16)])
def test_e2m1_round_trip(oracle_mod, codes):
    for c in codes:
        assert oracle_mod.e2m1_encode(oracle_mod.e2m1_decode(c)) == c


def test_e4m3_round_trip(oracle_mod):
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):
        assert oracle_mod.e4m3_encode(oracle_mod.e4m3_decode(c)) == c, hex(c)


def test_e2m1_midpoints_tie_to_even(oracle_mod):
    # midpoint -> code chosen (even code of the two neighbours)
    table = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in table.items():
        assert oracle_mod.e2m1_encode(v) == c
        assert oracle_mod.e2m1_encode(-v) == 8 | c
    assert oracle_mod.e2m1_encode(6.0001) == 7 and oracle_mod.e2m1_encode(1e30) == 7
    assert oracle_mod.e2m1_encode(-0.1) == 8 and oracle_mod.e2m1_encode(-0.0) == 8


def test_e4m3_saturation_and_underflow(oracle_mod):
    assert oracle_mod.e4m3_encode(448.0) == 0x7E
    assert oracle_mod.e4m3_encode(463.9) == 0x7E and oracle_mod.e4m3_encode(1e30) == 0x7E
    assert oracle_mod.e4m3_encode(2.0 ** -10) == 0          # tie between 0 and 2^-9
    assert oracle_mod.e4m3_encode(1.5 * 2.0 ** -9) == 2     # tie between 1 and 2
    assert oracle_mod.e4m3_encode(8.5) == 0x50              # tie between 8 and 9 -> 8


def _fnptr(lib, name):
    return ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


@pytest.mark.slow
def test_e2m1_encode_exhaustive(oracle_mod, brute):
    """Every binary32 bit pattern (NaNs skipped) against the brute-force search."""
    first = ctypes.c_uint32()
    bad = brute.brute_count_mismatch(_fnptr(oracle_mod._L(), "oracle_e2m1_encode"), 0,
                                     0, 1 << 32, ctypes.byref(first))
    assert bad == 0, f"{bad} mismatches, first pattern {first.value:#010x}"


@pytest.mark.slow
def test_e4m3_encode_exhaustive(oracle_mod, brute):
    """Every non-negative binary32 pattern up to +inf, plus every negative one."""
    first = ctypes.c_uint32()
    fn = _fnptr(oracle_mod._L(), "oracle_e4m3_encode")
    bad = brute.brute_count_mismatch(fn, 1, 0, 0x7F800001, ctypes.byref(first))
    assert bad == 0, f"{bad} mismatches, first pattern {first.value:#010x}"
    bad = brute.brute_count_mismatch(fn, 1, 0x80000000, 0xFF800001, ctypes.byref(first))
    assert bad == 0, f"{bad} negative mismatches, first pattern {first.value:#010x}"


def test_brute_force_checker_catches_a_planted_mistake(oracle_mod, brute):
    """The exhaustive checker must see a wrong tie rule: plant one on the CPU."""
    planted = ctypes.CFUNCTYPE(ctypes.c_uint8, ctypes.c_float)(
        lambda v: 1 if abs(v) == 0.25 else oracle_mod.e2m1_encode(v))
    first = ctypes.c_uint32()
    lo = 0x3E800000  # 0.25
    n = brute.brute_count_mismatch(ctypes.cast(planted, ctypes.c_void_p).value, 0,
                                   lo - 4, lo + 4, ctypes.byref(first))
    assert n == 1 and first.value == lo


def _bf16_exact(v: Fraction) -> Fraction:
    """bf16 round-to-nearest-even of an exact rational (normal range)."""
    if v == 0:
        return Fraction(0)
    a = abs(v)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (e - 7)
    n = a / q
    lo = math.floor(n)
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    r = lo * q
    return r if v > 0 else -r


def test_bf16_rne_against_torch(oracle_mod):
    """binary32 inputs: a single rounding to bf16 is torch's float->bf16 cast."""
    import torch
    rng = np.random.default_rng(1)
    f32 = rng.standard_normal(200_000).astype(np.float32) * np.float32(37.0)
    f32 = np.concatenate([f32, np.float32([1.00390625, 1.01171875, -3.00390625, 0.0, -0.0])])
    got = oracle_mod.bf16_rne_array(f32.astype(np.float64))
    want = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_bf16_rne_on_binary64_against_exact_rationals(oracle_mod):
    rnd = random.Random(5)
    for _ in range(3000):
        v = rnd.uniform(-1, 1) * 2.0 ** rnd.randint(-30, 30)
        bits = oracle_mod.bf16_rne(v)
        got = oracle_mod.bf16_to_f32(bits)
        assert Fraction(got) == _bf16_exact(Fraction(v)), v
    # ties just below/above: 1 + 2^-8 is a midpoint (-> 1), a hair above goes up
    assert oracle_mod.bf16_to_f32(oracle_mod.bf16_rne(1 + 2.0 ** -8)) == 1.0
    assert oracle_mod.bf16_to_f32(oracle_mod.bf16_rne(1 + 2.0 ** -8 + 2.0 ** -40)) == 1 + 2.0 ** -7
