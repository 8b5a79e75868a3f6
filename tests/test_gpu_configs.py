"""GPU parity of the W4A4 linear (mq_linear_w4a4, the launch configuration
bench.py times) at the full sizes of the workloads it stands for, on sampled
output rows the CPU oracle computes in full:

  * long-context prefill: 32768 tokens, heavy-tailed activations (Student-t,
    nu = 4, per-channel LogNormal scale), the four Qwen3-8B-shaped projections;
  * the 131072-token projections of a Qwen3-8B-shaped decoder layer (qkv,
    gate/up; o and down are in the sweep);
  * the shape sweep: tokens M in {512, 2048, 8192, 32768, 131072} x (K, N) in
    {(4096, 4096), (4096, 12288), (12288, 4096), (5120, 25600)}.

alpha_x is checked against the oracle on the whole activation (it depends on
every element), the output rows are independent of each other, so a sample of
rows checks the GEMM at full size.  Tolerance: relative Frobenius error
<= 1e-3 against the oracle's exact product of the dequantized operands
rounded to bf16 (NVFP4 W4A4: "Mix-Quant：面向智能体LLM的量化预填充与精确解码",
section 方法步骤详情, step (3)).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import bits, check_gemm_elementwise, dev, linear_ws_codes_rows, linear_ws_scales

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
TOL = 1e-3


def _sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    rows = np.random.default_rng(seed).choice(M, min(n, M), replace=False)
    return np.unique(np.concatenate([rows, [0, M - 1]]))


def _host_bits_chunked(x: torch.Tensor, chunk_rows: int = 8192) -> np.ndarray:
    """bf16 bit patterns of a device tensor, copied to the host in chunks."""
    out = np.empty(x.shape, np.uint16)
    for r in range(0, x.shape[0], chunk_rows):
        out[r:r + chunk_rows] = bits(x[r:r + chunk_rows])
    return out


def _check_linear(x_dev: torch.Tensor, w_dev: torch.Tensor, rows: np.ndarray):
    """Run mq_linear_w4a4 on (x, w) and compare the sampled rows of Y and the
    activation's alpha (whole tensor) with the oracle."""
    M, K = x_dev.shape
    N = w_dev.shape[0]
    lin = mq.LinearW4A4(w_dev)
    y = lin(x_dev)
    torch.cuda.synchronize()
    assert mq.mq_read_status(lin._ws) == mq.MQ_OK
    xb = _host_bits_chunked(x_dev)
    wb = _host_bits_chunked(w_dev)
    ax = oracle.tensor_scale(xb)
    aw = oracle.tensor_scale(wb)
    assert float(lin.w.alpha.item()) == aw
    # alpha_x as the linear computed it: word 3 of the workspace header (the
    # library's layout: amax bits, ticket, status, alpha, generation)
    alpha_linear = float(lin._ws[12:16].view(torch.float32).item())
    assert alpha_linear == ax, (alpha_linear, ax)
    # and through the public calls (k_amax rather than the one-pass kernel)
    qx = mq.quantize(x_dev)
    torch.cuda.synchronize()
    assert float(qx.alpha.item()) == ax
    del qx
    xc, xs = oracle.quantize(np.ascontiguousarray(xb[rows]), ax)
    # the linear's own quantized activation on those rows, bit for bit
    ws_codes = linear_ws_codes_rows(lin._ws, M, K, rows)
    bad = np.argwhere(ws_codes != xc)
    assert len(bad) == 0, f"{len(bad)} code bytes differ, first {bad[:4].tolist()}"
    ws_scales = oracle.scales_from_stored(linear_ws_scales(lin._ws, M, K), M, K)[rows]
    bad = np.argwhere(ws_scales != xs)
    assert len(bad) == 0, f"{len(bad)} scales differ, first {bad[:4].tolist()}"
    wc, wsc = oracle.quantize(wb, aw)
    got = bits(y[torch.from_numpy(rows).to(y.device)])
    _, err = check_gemm_elementwise(got, oracle.dequantize(xc, xs, ax), oracle.dequantize(wc, wsc, aw), K)
    assert err <= TOL, err
    return err


@pytest.mark.parametrize("proj", inputs.QWEN3_8B_PROJECTIONS, ids=lambda p: p.name)
def test_long_context_32k_student_t(proj):
    M, K, N = 32768, proj.K, proj.N
    x = inputs.student_t_activation_bf16(M, K, seed=300 + K).to(dev())
    w = inputs.weight_bf16(N, K, seed=400 + N, device="cuda")
    _check_linear(x, w, _sample_rows(M, 96, seed=K + N))


_SWEEP = [(M, K, N) for M in inputs.SWEEP_M for (K, N) in inputs.SWEEP_KN]
_LAYER_131K = [(131072, p.K, p.N) for p in inputs.QWEN3_8B_PROJECTIONS if p.name in ("qkv", "gate_up")]


@pytest.mark.parametrize("M,K,N", _SWEEP + _LAYER_131K, ids=lambda v: str(v))
def test_full_size_sampled_rows(M, K, N):
    x = inputs.activation_bf16(M, K, seed=M % 9973 + K, outlier_channels=inputs.outlier_count(K),
                               outlier_scale=50.0, device="cuda")
    w = inputs.weight_bf16(N, K, seed=N + 7, device="cuda")
    _check_linear(x, w, _sample_rows(M, 48, seed=M + K + N))
