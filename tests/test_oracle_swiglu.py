"""Pins of the oracle's SwiGLU, the activation between the MLP's gate/up and
down W4A4 linears (the pages quantize both linears, "Mix-Quant：面向智能体LLM的
量化预填充与精确解码", section 方法步骤详情, step (3); they give the gated
activation no numerics, so its binary32 form is a reading: R11-R13 in the
oracle's source).

Pins, none of which re-types the oracle's formula:
  * the binary32 exponential against the binary64 library exponential, within
    2 units in the last place over a dense sweep, and exact where e^x is a
    power of two times an exactly known value (x = 0);
  * silu(g) for every finite bf16 g against g / (1 + e^-g) in binary64, within
    4 units in the last place, plus its limits (silu(0) = 0, silu(g) = g for
    large g, -0 for very negative g);
  * h = bf16(silu(g) u) against the binary64 value rounded to bf16: equal, or
    one bf16 step apart only where the binary64 value lies within 2^-20 of a
    bf16 rounding midpoint;
  * the gate/up split of the composite MLP reference on a construction whose
    gate and up products are known exactly (a swapped split fails it).
"""
import math

import numpy as np
import pytest

from nvfp4_w4a4_quantized_03_b200 import inputs


def _ulp32(v: float) -> float:
    v = abs(v)
    if v == 0.0:
        return 2.0 ** -149
    e = math.frexp(v)[1] - 1
    return 2.0 ** (max(e, -126) - 23)


def test_exp_against_binary64(oracle_mod):
    xs = np.concatenate([np.linspace(-87.0, 88.0, 40001), np.random.default_rng(7).uniform(-87, 88, 20000),
                         np.linspace(-1, 1, 2001)]).astype(np.float32)
    worst = 0.0
    for x in xs.tolist():
        got = oracle_mod.exp_f32(x)
        ref = math.exp(x)
        worst = max(worst, abs(got - ref) / _ulp32(ref))
    assert worst <= 2.0, worst
    assert oracle_mod.exp_f32(0.0) == 1.0
    assert oracle_mod.exp_f32(100.0) == math.inf
    assert oracle_mod.exp_f32(-100.0) == 0.0


def _all_finite_bf16() -> np.ndarray:
    b = np.arange(65536, dtype=np.uint32)
    exp = (b >> 7) & 0xFF
    return b[exp != 0xFF].astype(np.uint16)


def _bf16_value(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_silu_every_bf16_input(oracle_mod):
    g = _bf16_value(_all_finite_bf16())
    worst = 0.0
    for v in g.tolist():
        got = oracle_mod.silu_f32(v)
        if v < -88.0:
            # e(-g) is +inf there: silu is -0 (the true value is below 2^-120 in magnitude)
            assert got == 0.0 and math.copysign(1.0, got) < 0
            continue
        ref = v / (1.0 + math.exp(-v))
        if ref == 0.0:
            assert got == 0.0
            continue
        worst = max(worst, abs(got - ref) / _ulp32(ref))
    assert worst <= 4.0, worst
    assert oracle_mod.silu_f32(0.0) == 0.0
    assert oracle_mod.silu_f32(200.0) == 200.0
    assert oracle_mod.silu_f32(-1.0) < 0 and abs(oracle_mod.silu_f32(-1.0) - (-1.0 / (1.0 + math.e))) < 1e-7


def _bf16_rne_f64(v: np.ndarray) -> np.ndarray:
    """Round binary64 values to bf16 values (nearest, ties to even), in numpy."""
    out = np.empty_like(v)
    for i, x in enumerate(v.tolist()):
        if x == 0.0 or not math.isfinite(x):
            out[i] = x
            continue
        e = math.frexp(abs(x))[1] - 1
        q = 2.0 ** (max(e, -126) - 7)
        n = x / q
        r = math.floor(n)
        d = n - r
        if d > 0.5 or (d == 0.5 and r % 2 == 1):
            r += 1
        out[i] = math.copysign(math.inf, x) if abs(r * q) >= 2.0 ** 128 else r * q
    return out


@pytest.mark.parametrize("u", [1.0, -0.75, 3.140625, 1e-3])
def test_swiglu_rounding(oracle_mod, u):
    gbits = _all_finite_bf16()
    g = _bf16_value(gbits)
    ubits = np.full(gbits.shape, oracle_mod.bf16_rne(u), np.uint16)
    uval = _bf16_value(ubits)
    h = _bf16_value(oracle_mod.swiglu_bf16(gbits, ubits))
    with np.errstate(over="ignore"):
        exact = np.where(g < -88.0, -0.0 * uval, g / (1.0 + np.exp(-g)) * uval)
    ref = _bf16_rne_f64(exact)
    differ = h != ref
    # a difference is allowed only next to a bf16 rounding midpoint, and only by one step
    for i in np.nonzero(differ)[0].tolist():
        x = exact[i]
        if math.isinf(h[i]):
            # binary32 overflow: the exact value is at least the largest finite
            # bf16 plus half a step, within binary32 rounding
            assert abs(x) >= (2.0 ** 128 - 2.0 ** 120) * (1 - 2.0 ** -20), (g[i], x)
            continue
        e = math.frexp(abs(x))[1] - 1
        q = 2.0 ** (max(e, -126) - 7)
        frac = abs(x) / q - math.floor(abs(x) / q)
        assert abs(frac - 0.5) < 2.0 ** -20 * abs(x) / q + 2 ** -30, (g[i], x, h[i], ref[i])
        assert abs(h[i] - ref[i]) <= q * 1.0000001
    # (where 1 + e^-g rounds to 1 in binary32, silu(g) u can sit exactly on a
    # midpoint that the binary64 value misses by far less than 2^-20)


def test_swiglu_signs_and_limits(oracle_mod):
    one = oracle_mod.bf16_rne(1.0)
    # g = 0 -> +0; very negative g -> -0 times u; large g -> g * u
    h = oracle_mod.swiglu_bf16(np.array([0x0000, oracle_mod.bf16_rne(-100.0), oracle_mod.bf16_rne(100.0)], np.uint16),
                               np.array([one, one, oracle_mod.bf16_rne(2.0)], np.uint16))
    assert h.tolist() == [0x0000, 0x8000, oracle_mod.bf16_rne(200.0)]


def test_gate_up_split(oracle_mod):
    """x = all ones, gate rows all equal to a, up rows all equal to b (a and b
    exact in NVFP4; xhat = 1 within 2^-25): every gate product rounds to the
    bf16 value K a and every up product to K b, so h = swiglu(K a, K b);
    silu(K a) K b differs from silu(K b) K a, so a swapped split fails."""
    M, K, inter = 3, 64, 16
    x = np.full((M, K), oracle_mod.bf16_rne(1.0), np.uint16)
    a, b = 0.25, -0.0625          # K a = 16, K b = -4
    w = np.zeros((2 * inter, K), np.uint16)
    w[:inter] = oracle_mod.bf16_rne(a)
    w[inter:] = oracle_mod.bf16_rne(b)
    ref = oracle_mod.mlp_w4a4(x, w, np.full((16, inter), oracle_mod.bf16_rne(1.0), np.uint16))
    assert np.all(ref["g"] == oracle_mod.bf16_rne(K * a))
    assert np.all(ref["u"] == oracle_mod.bf16_rne(K * b))
    want = oracle_mod.bf16_rne(16.0 / (1.0 + math.exp(-16.0)) * -4.0)
    assert np.all(ref["h"] == want)
    swapped = oracle_mod.bf16_rne(-4.0 / (1.0 + math.exp(4.0)) * 16.0)
    assert want != swapped


def test_mlp_reference_on_random_inputs(oracle_mod):
    """The composite on seeded inputs: alpha_h is max|h| / 2688 of the H it
    returns, and the down product is the quantized H times the quantized W_d."""
    M, K, inter, N = 8, 128, 128, 64
    x = inputs.bf16_bits(inputs.activation_bf16(M, K, seed=5, outlier_channels=2, outlier_scale=20.0))
    wgu = inputs.bf16_bits(inputs.weight_bf16(2 * inter, K, seed=6))
    wd = inputs.bf16_bits(inputs.weight_bf16(N, inter, seed=7))
    ref = oracle_mod.mlp_w4a4(x, wgu, wd)
    hmax = np.max(np.abs(_bf16_value(ref["h"])))
    assert ref["alpha_h"] == float(np.float32(np.float32(hmax) / np.float32(2688.0)))
    assert ref["y64"].shape == (M, N)
