"""Pins of the oracle's contraction and of the block-scale storage order.

The W4A4 linear is Y = bf16(xhat . what^T) with xhat = alpha_x sigma_b q
("Mix-Quant：面向智能体LLM的量化预填充与精确解码", section 方法步骤详情, step (3);
r9-hu digest, section Method, item 1, both operands quantized: W4A4).
Pins: exact rational brute force on small shapes, an identity weight, and
hand-computed offsets of the scale storage order.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_03_b200 import inputs


def _exact_product(xh, wh):
    M, K = xh.shape
    N = wh.shape[0]
    xf = [[Fraction(v) for v in row] for row in xh]
    wf = [[Fraction(v) for v in row] for row in wh]
    return [[sum(a * b for a, b in zip(xf[m], wf[n])) for n in range(N)] for m in range(M)]


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (3, 17, 64), (17, 3, 128), (5, 9, 128)])
def test_gemm_against_exact_rationals(oracle_mod, M, N, K):
    x = inputs.activation_bf16(M, K, seed=M * 100 + N, outlier_channels=2, outlier_scale=20.0)
    w = inputs.weight_bf16(N, K, seed=K + N)
    ref = oracle_mod.linear_w4a4(inputs.bf16_bits(x), inputs.bf16_bits(w))
    xh = oracle_mod.dequantize(ref["x_codes"], ref["x_scales"], ref["alpha_x"])
    wh = oracle_mod.dequantize(ref["w_codes"], ref["w_scales"], ref["alpha_w"])
    exact = _exact_product(xh, wh)
    absdot = np.abs(xh) @ np.abs(wh).T
    for m, n in itertools.product(range(M), range(N)):
        e = exact[m][n]
        got = ref["y64"][m, n]
        # binary64 summation bound: K * 2^-53 * sum |a_k b_k|
        assert abs(Fraction(got) - e) <= Fraction(float(absdot[m, n])) * K * Fraction(1, 2 ** 52)
        # bf16 of the product: unique unless the exact value sits on a bf16 midpoint
        ybits = ref["y_bf16"][m, n]
        yv = Fraction(oracle_mod.bf16_to_f32(int(ybits)))
        if e != 0:
            assert abs(yv - e) <= abs(e) * Fraction(1, 256)


def test_gemm_identity_weight_reproduces_xhat(oracle_mod):
    """W = 6 * I with exact scales: Y = bf16(xhat * alpha_w * sigma_w * 6)."""
    K = 128
    x = inputs.activation_bf16(8, K, seed=4, outlier_channels=3, outlier_scale=30.0)
    w = torch.eye(K, dtype=torch.bfloat16) * 6.0
    ref = oracle_mod.linear_w4a4(inputs.bf16_bits(x), inputs.bf16_bits(w))
    # alpha_w = 6 / 2688 and every block scale is 448, so what = 6 * I exactly
    wh = oracle_mod.dequantize(ref["w_codes"], ref["w_scales"], ref["alpha_w"])
    assert np.allclose(wh, 6.0 * np.eye(K), rtol=2 ** -22, atol=0)
    xh = oracle_mod.dequantize(ref["x_codes"], ref["x_scales"], ref["alpha_x"])
    assert np.array_equal(ref["y_bf16"], oracle_mod.bf16_rne_array(xh @ wh.T))


def test_scale_offsets_by_hand(oracle_mod):
    # K = 256: 16 scale columns = 4 k-atoms per row tile
    K = 256
    f = oracle_mod.scale_offset
    assert f(0, 0, K) == 0
    assert f(0, 1, K) == 1            # next scale column, same 32-bit word
    assert f(1, 0, K) == 16           # next row: 16 bytes further
    assert f(32, 0, K) == 4           # row 32 shares row 0's 16 bytes, word 1
    assert f(96, 3, K) == 15
    assert f(31, 0, K) == 496
    assert f(0, 4, K) == 512          # second k-atom of row tile 0
    assert f(0, 15, K) == 3 * 512 + 3
    assert f(128, 0, K) == 4 * 512    # row tile 1 follows all k-atoms of tile 0
    assert f(200, 9, K) == 4 * 512 + 2 * 512 + (200 % 32) * 16 + ((200 // 32) % 4) * 4 + 1


@pytest.mark.parametrize("rows,K", [(1, 64), (130, 128), (256, 1024), (77, 320)])
def test_scale_storage_is_a_bijection(oracle_mod, rows, K):
    nb = K // 16
    padded_rows = -(-rows // 128) * 128
    padded_nb = -(-nb // 4) * 4
    assert oracle_mod.scale_bytes(rows, K) == padded_rows * padded_nb
    offs = {oracle_mod.scale_offset(r, b, K) for r in range(padded_rows) for b in range(padded_nb)}
    assert offs == set(range(padded_rows * padded_nb))
    rng = np.random.default_rng(rows)
    logical = rng.integers(1, 255, size=(rows, nb), dtype=np.uint8)
    stored = oracle_mod.scales_to_stored(logical, K)
    assert np.array_equal(oracle_mod.scales_from_stored(stored, rows, K), logical)
    assert (stored != 0).sum() == rows * nb       # padding stays zero
