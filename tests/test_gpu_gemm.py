"""GPU parity of the block-scaled FP4 GEMM (mq_nvfp4_gemm) and of the fused
linear (mq_linear_w4a4) against the CPU oracle.

Y = bf16(xhat . what^T), xhat = alpha sigma q ("Mix-Quant：面向智能体LLM的量化预填充
与精确解码", section 方法步骤详情, step (3); W4A4).  Tolerance: relative
Frobenius error <= 1e-3 against the oracle's bf16 result on the same quantized
operands, and on every element the bound of gpu_helpers.check_elementwise
(the two bf16 roundings plus the worst-case binary32 accumulation error of a
K-term sum); bit-exact where every partial sum is exact in binary32.  The
linear's own quantized activation (the codes and scales mq_linear_w4a4 leaves
in its workspace) is compared with the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import (bits, check_gemm_elementwise, dev, gpu_quantize, linear_ws_codes_rows, linear_ws_offsets, linear_ws_scales)

pytestmark = pytest.mark.gpu
TOL = 1e-3


@pytest.fixture(params=["auto", "1", "2"])
def gemm_form(request, switches):
    """Run a test with the library's choice of GEMM form, then forced to each
    of: one CTA (128 x 256 tiles) or a CTA pair (256 x 256 tiles)."""
    if request.param != "auto":
        switches(gemm_form=int(request.param))
    return request.param


def _gemm(qa, qb, M, N, K):
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    mq.mq_nvfp4_gemm(qa.codes, qa.scales, qa.alpha, qb.codes, qb.scales, qb.alpha, M, N, K, y, ws)
    torch.cuda.synchronize()
    assert mq.mq_read_status(ws) == mq.MQ_OK
    return bits(y)


def _upload(codes_np, logical_scales, K, alpha):
    rows = codes_np.shape[0]
    q = mq.QuantizedTensor(rows, K, dev())
    q.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes_np).reshape(-1)))
    q.scales.copy_(torch.from_numpy(oracle.scales_to_stored(logical_scales, K)))
    q.alpha.fill_(alpha)
    return q


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (128, 256, 256), (200, 300, 512), (1, 8, 64), (257, 513, 320),
                                   (512, 512, 256)])
def test_exact_products_bit_exact(M, N, K, gemm_form):
    """Codes random, scales powers of two in [2^-2, 2^2], alpha = 1: every
    partial sum is exact in binary32, so Y must equal the oracle bit for bit.
    Pins the MMA's reading of code nibbles, E4M3 scales and the scale order."""
    rng = np.random.default_rng(M * 7 + N + K)
    pow2 = np.array([(e + 7) << 3 for e in range(-2, 3)], np.uint8)   # E4M3 codes of 2^e
    ac = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    bc = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    asc = pow2[rng.integers(0, 5, size=(M, K // 16))]
    bsc = pow2[rng.integers(0, 5, size=(N, K // 16))]
    y = _gemm(_upload(ac, asc, K, 1.0), _upload(bc, bsc, K, 1.0), M, N, K)
    ref = oracle.bf16_rne_array(oracle.gemm_f64(oracle.dequantize(ac, asc, 1.0), oracle.dequantize(bc, bsc, 1.0)))
    bad = np.argwhere(y != ref)
    assert len(bad) == 0, f"{len(bad)} mismatches, first {bad[:4].tolist()}"


def test_alpha_product_scaling():
    """alpha_a * alpha_b (powers of two) scales Y exactly."""
    M, N, K = 128, 256, 128
    rng = np.random.default_rng(3)
    ac = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    bc = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sc = np.full((M, K // 16), 0x38, np.uint8)   # 1.0
    sb = np.full((N, K // 16), 0x38, np.uint8)
    y = _gemm(_upload(ac, sc, K, 2.0 ** -3), _upload(bc, sb, K, 2.0 ** 5), M, N, K)
    ref = oracle.bf16_rne_array(4.0 * oracle.gemm_f64(oracle.dequantize(ac, sc, 1.0), oracle.dequantize(bc, sb, 1.0)))
    assert np.array_equal(y, ref)


def _random_case(M, N, K, seed, student_t=False):
    if student_t:
        x = inputs.student_t_activation_bf16(M, K, seed=seed)
    else:
        x = inputs.activation_bf16(M, K, seed=seed, outlier_channels=max(1, inputs.outlier_count(K)),
                                   outlier_scale=50.0)
    w = inputs.weight_bf16(N, K, seed=seed + 1000)
    return x, w


@pytest.mark.parametrize("M,N,K", [(128, 1024, 1024), (1, 256, 64), (3, 17, 128), (17, 3, 64), (130, 300, 320),
                                   (257, 513, 1024), (300, 257, 128), (512, 1024, 4096), (96, 4096, 12288)])
def test_gemm_random_against_oracle(M, N, K, gemm_form):
    x, w = _random_case(M, N, K, seed=M + N + K)
    ax, xc, xs, qx = gpu_quantize(x)
    aw, wc, wsc, qw = gpu_quantize(w)
    y = _gemm(qx, qw, M, N, K)
    ref = oracle.linear_w4a4(bits(x), bits(w))
    assert ref["alpha_x"] == ax and ref["alpha_w"] == aw
    assert np.array_equal(ref["x_codes"], xc) and np.array_equal(ref["w_codes"], wc)
    _, err = check_gemm_elementwise(y, oracle.dequantize(ref["x_codes"], ref["x_scales"], ax),
                                    oracle.dequantize(ref["w_codes"], ref["w_scales"], aw), K)
    assert err <= TOL, err


def test_linear_equals_separate_calls_and_oracle():
    M, N, K = 200, 768, 1024
    x, w = _random_case(M, N, K, seed=5, student_t=True)
    qw = mq.quantize(w.to(dev()))
    _, _, _, qx = gpu_quantize(x)
    y_sep = _gemm(qx, qw, M, N, K)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
    ws = mq.workspace(mq.mq_linear_w4a4_workspace_bytes(M, K), dev())
    for _ in range(2):      # the workspace is reusable call after call
        mq.mq_linear_w4a4(x.to(dev()), qw.codes, qw.scales, qw.alpha, N, y, ws)
        torch.cuda.synchronize()
        assert mq.mq_read_status(ws) == mq.MQ_OK
        assert np.array_equal(bits(y), y_sep)
    ref = oracle.linear_w4a4(bits(x), bits(w))
    _check_linear_ws(ws, ref, M, K)
    _, err = check_gemm_elementwise(bits(y), oracle.dequantize(ref["x_codes"], ref["x_scales"], ref["alpha_x"]),
                                    oracle.dequantize(ref["w_codes"], ref["w_scales"], ref["alpha_w"]), K)
    assert err <= TOL


def _check_linear_ws(ws, ref, M, K, rows=None):
    """The quantized activation the linear left in its workspace equals the
    oracle's codes and scales bit for bit: all rows, or the rows given (ref
    then holds the oracle's codes and scales of those rows, in order)."""
    codes = linear_ws_codes_rows(ws, M, K, rows)
    bad = np.argwhere(codes != ref["x_codes"])
    assert len(bad) == 0, f"{len(bad)} code bytes differ, first {bad[:4].tolist()}"
    scales = oracle.scales_from_stored(linear_ws_scales(ws, M, K), M, K)
    if rows is not None:
        scales = scales[rows]
    bad = np.argwhere(scales != ref["x_scales"])
    assert len(bad) == 0, f"{len(bad)} scales differ, first {bad[:4].tolist()}"
    if rows is None:
        # the padding rows of the stored scales are zero
        stored = linear_ws_scales(ws, M, K)
        assert np.array_equal(oracle.scales_to_stored(scales, K), stored)


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (130, 300, 320), (257, 513, 1024), (700, 1024, 4096),
                                   (128, 256, 12288), (2100, 768, 2048)])
@pytest.mark.parametrize("form", ["auto", "1", "2"])
def test_linear_paths_agree(M, N, K, form, switches):
    """The three ways mq_linear_w4a4 can quantize X -- the one-pass
    cooperative quantizer (default), the tensor-scale + quantize kernels, and
    quantizer warps inside the GEMM -- give the same Y bit for bit, and the
    oracle's within tolerance."""
    if form != "auto":
        switches(gemm_form=int(form))
    x, w = _random_case(M, N, K, seed=M + 3 * N + K, student_t=(M % 2 == 0))
    qw = mq.quantize(w.to(dev()))
    xd = x.to(dev())
    ws = mq.workspace(mq.mq_linear_w4a4_workspace_bytes(M, K), dev())
    ref = oracle.linear_w4a4(bits(x), bits(w))
    outs = []
    for path in ("onepass", "split", "ingemm", "onepass"):
        switches(linear_path=path)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev())
        ws[linear_ws_offsets(M, K)[0]:].fill_(0x5A)      # stale bytes where the quantized activation goes
        mq.mq_linear_w4a4(xd, qw.codes, qw.scales, qw.alpha, N, y, ws)
        torch.cuda.synchronize()
        assert mq.mq_read_status(ws) == mq.MQ_OK
        _check_linear_ws(ws, ref, M, K)
        outs.append(bits(y))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    _, err = check_gemm_elementwise(outs[0], oracle.dequantize(ref["x_codes"], ref["x_scales"], ref["alpha_x"]),
                                    oracle.dequantize(ref["w_codes"], ref["w_scales"], ref["alpha_w"]), K)
    assert err <= TOL


@pytest.mark.slow
@pytest.mark.parametrize("proj", inputs.QWEN3_8B_PROJECTIONS, ids=lambda p: p.name)
def test_prefill_projection_8k_sampled_rows(proj):
    """Full 8192-token projections through mq_linear_w4a4; the oracle checks
    alpha on the whole activation and 256 sampled output rows in full."""
    M, K, N = 8192, proj.K, proj.N
    x, w = _random_case(M, N, K, seed=17)
    lin = mq.LinearW4A4(w.to(dev()))
    y = lin(x.to(dev()))
    torch.cuda.synchronize()
    assert mq.mq_read_status(lin._ws) == mq.MQ_OK
    xb, wb = bits(x), bits(w)
    ax = oracle.tensor_scale(xb)
    aw = oracle.tensor_scale(wb)
    assert float(lin.w.alpha.item()) == aw
    # the whole quantized activation the linear wrote, bit for bit
    xc_all, xs_all = oracle.quantize(xb, ax)
    _check_linear_ws(lin._ws, dict(x_codes=xc_all, x_scales=xs_all), M, K)
    rows = np.sort(np.random.default_rng(0).choice(M, 256, replace=False))
    wc, wsc = oracle.quantize(wb, aw)
    got = bits(y)[rows]
    _, err = check_gemm_elementwise(got, oracle.dequantize(xc_all[rows], xs_all[rows], ax),
                                    oracle.dequantize(wc, wsc, aw), K)
    assert err <= TOL


def test_raster_groups_with_a_ragged_last_group(switches):
    """At K = 16384 a raster group holds at most 18 MiB of A, i.e. 7 M-blocks
    of 256 rows, so M = 2900 (12 M-blocks) runs as one group of 7 and a
    ragged one of 5.  Every tile computes the same sums whatever the order of
    the tiles: Y equals the one-M-block-per-group raster's bit for bit, and
    the oracle on sampled rows within the per-element bound."""
    M, N, K = 2900, 520, 16384
    x, w = _random_case(M, N, K, seed=77)
    ax, xc, xs, qx = gpu_quantize(x)
    aw, wc, wsc, qw = gpu_quantize(w)
    y = _gemm(qx, qw, M, N, K)
    switches(gemm_group_m=1)
    assert np.array_equal(_gemm(qx, qw, M, N, K), y)
    rows = np.sort(np.random.default_rng(5).choice(M, 96, replace=False))
    rows = np.union1d(rows, [0, 255, 256, 1791, 1792, 2899])          # group and block edges
    assert oracle.tensor_scale(bits(x)) == ax and oracle.tensor_scale(bits(w)) == aw
    x_codes, x_scales = oracle.quantize(bits(x)[rows], ax)
    w_codes, w_scales = oracle.quantize(bits(w), aw)
    assert np.array_equal(x_codes, xc[rows]) and np.array_equal(w_codes, wc)
    _, err = check_gemm_elementwise(y[rows], oracle.dequantize(x_codes, x_scales, ax),
                                    oracle.dequantize(w_codes, w_scales, aw), K)
    assert err <= TOL, err
