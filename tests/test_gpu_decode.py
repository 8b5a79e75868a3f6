"""GPU parity of the decode-shaped GEMM (few rows of A: mq_nvfp4_gemm and
mq_linear_w4a4 take the weight-streaming split-K kernel for M <= 64) against
the CPU oracle and against the prefill-shaped kernel.

Y = bf16(xhat . what^T), xhat = alpha sigma q (NVFP4 W4A4, "Mix-Quant：面向
智能体LLM的量化预填充与精确解码", section 方法步骤详情, step (3); decoding
quantized as well is the pages' P16D4 variant).  Tolerance: relative
Frobenius error <= 1e-3 against the oracle's bf16 result on the same
quantized operands, and the per-element bound of
gpu_helpers.check_elementwise on every output.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import bf16_bits_to_f64, bits, check_gemm_elementwise, dev, gpu_quantize, rel_frobenius

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _check_against_oracle(got, xb, wb):
    """Per-element bound and relative Frobenius error of a GEMM output against
    the oracle on the oracle's quantization of (x, w)."""
    ax, aw = oracle.tensor_scale(xb), oracle.tensor_scale(wb)
    xc, xs = oracle.quantize(xb, ax)
    wc, wsc = oracle.quantize(wb, aw)
    _, err = check_gemm_elementwise(got, oracle.dequantize(xc, xs, ax), oracle.dequantize(wc, wsc, aw),
                                    xb.shape[1])
    assert err <= TOL, err


def _gemm(M, N, K, x, w):
    _, _, _, qx = gpu_quantize(x)
    _, _, _, qw = gpu_quantize(w)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev())
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, qw.codes, qw.scales, qw.alpha, M, N, K, y, ws)
    torch.cuda.synchronize()
    assert mq.mq_read_status(ws) == mq.MQ_OK
    return bits(y)


@pytest.mark.parametrize("M", [1, 2, 7, 16, 17, 33, 64])
@pytest.mark.parametrize("N,K", [(4096, 4096), (130, 320), (6144, 4096), (300, 12288), (24576, 1024)])
@pytest.mark.parametrize("split", ["auto", "1", "8"])
def test_decode_gemm_against_oracle(M, N, K, split, switches):
    if split != "auto":
        switches(decode_split=int(split))
    x = inputs.activation_bf16(M, K, seed=M * 7 + K, outlier_channels=max(1, inputs.outlier_count(K)),
                               outlier_scale=50.0)
    w = inputs.weight_bf16(N, K, seed=N + 3)
    got = _gemm(M, N, K, x, w)
    _check_against_oracle(got, bits(x), bits(w))


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 12288, 4096), (64, 4096, 12288)])
def test_decode_matches_prefill_kernel(M, N, K, switches):
    """The split-K kernel and the prefill-shaped kernel differ only in the
    order of the fp32 additions."""
    x = inputs.student_t_activation_bf16(M, K, seed=M + K)
    w = inputs.weight_bf16(N, K, seed=K + 1)
    a = _gemm(M, N, K, x, w)
    switches(gemm_decode=0)
    b = _gemm(M, N, K, x, w)
    assert rel_frobenius(bf16_bits_to_f64(a), bf16_bits_to_f64(b)) <= TOL
    _check_against_oracle(a, bits(x), bits(w))
    _check_against_oracle(b, bits(x), bits(w))


@pytest.mark.parametrize("M", [1, 8, 64])
def test_decode_linear(M):
    """mq_linear_w4a4 on a decode batch (quantize X, then the split-K GEMM)."""
    K, N = 4096, 6144
    x = inputs.activation_bf16(M, K, seed=M, outlier_channels=41, outlier_scale=50.0)
    w = inputs.weight_bf16(N, K, seed=5)
    lin = mq.LinearW4A4(w.to(dev()))
    y = lin(x.to(dev()))
    torch.cuda.synchronize()
    assert mq.mq_read_status(lin._ws) == mq.MQ_OK
    _check_against_oracle(bits(y), bits(x), bits(w))
