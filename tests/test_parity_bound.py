"""The per-element bound the GPU parity tests apply (gpu_helpers.check_elementwise)
checked on the CPU: it holds for a binary32 accumulation of the oracle's
quantized operands in two different summation orders, and it catches a
single wrong output element that the relative Frobenius error of the whole
output (1e-3) lets through."""
import numpy as np
import pytest

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs
from tests.gpu_helpers import check_elementwise, gemm_bound_terms, rel_frobenius, bf16_bits_to_f64

M, N, K = 256, 256, 1024


def _operands():
    x = inputs.activation_bf16(M, K, seed=3, outlier_channels=10, outlier_scale=50.0)
    w = inputs.weight_bf16(N, K, seed=4)
    xb = x.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    wb = w.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    ax, aw = oracle.tensor_scale(xb), oracle.tensor_scale(wb)
    xc, xs = oracle.quantize(xb, ax)
    wc, wsc = oracle.quantize(wb, aw)
    # sigma * q per operand (exact in binary32), and the alphas
    return (oracle.dequantize(xc, xs, 1.0), oracle.dequantize(wc, wsc, 1.0), ax, aw)


def _binary32_linear(a, w, ax, aw, reverse):
    """y = bf16(fl32(fl32(ax aw) * acc)) with acc the binary32 running sum of
    the K products (each exact in binary32), in k order or reversed."""
    a32, w32 = a.astype(np.float32), w.astype(np.float32)
    acc = np.zeros((M, N), np.float32)
    ks = range(K - 1, -1, -1) if reverse else range(K)
    for k in ks:
        acc = (acc + np.outer(a32[:, k], w32[:, k]).astype(np.float32)).astype(np.float32)
    y32 = (np.float32(np.float32(ax) * np.float32(aw)) * acc).astype(np.float32)
    return oracle.bf16_rne_array(y32.astype(np.float64))


@pytest.mark.parametrize("reverse", [False, True])
def test_bound_holds_for_binary32_accumulation(reverse):
    a, w, ax, aw = _operands()
    y = _binary32_linear(a, w, ax, aw, reverse)
    y64, _, acc = gemm_bound_terms(a * ax, w * aw, K)
    stats = check_elementwise(y, oracle.bf16_rne_array(y64), acc)
    assert stats["frac_differ"] > 0          # the two sides do round differently somewhere


def test_bound_catches_one_element_the_norm_misses():
    a, w, ax, aw = _operands()
    y = _binary32_linear(a, w, ax, aw, False)
    y64, _, acc = gemm_bound_terms(a * ax, w * aw, K)
    ref = oracle.bf16_rne_array(y64)
    i = np.unravel_index(int(np.argmax(np.abs(y64))), y64.shape)
    bad = bf16_bits_to_f64(y)
    bad[i] += 0.5e-3 * np.linalg.norm(bf16_bits_to_f64(ref))       # half the norm's tolerance on one element
    bad_bits = oracle.bf16_rne_array(bad)
    assert rel_frobenius(bf16_bits_to_f64(bad_bits), bf16_bits_to_f64(ref)) <= 1e-3
    with pytest.raises(AssertionError):
        check_elementwise(bad_bits, ref, acc)
