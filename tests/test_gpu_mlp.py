"""GPU parity of the W4A4 MLP: the gate/up GEMM with SwiGLU in its epilogue
(mq_nvfp4_gemm_swiglu) and the whole chain (mq_mlp_w4a4: quantize x, gate/up
GEMM + SwiGLU + max|h|, alpha_h, quantize H, down GEMM).

Both linears are NVFP4 W4A4 ("Mix-Quant：面向智能体LLM的量化预填充与精确解码",
section 方法步骤详情, step (3)); the gated activation between them follows the
oracle's readings R11-R13 (bf16 G and U, binary32 SwiGLU, H quantized with its
own tensor scale).

  * bit-exact: operands whose products and partial sums are exact in
    binary32 (random codes, power-of-two scales), so G and U are the oracle's
    and H, max|h| and H's NVFP4 form must match it bit for bit;
  * tolerance on realistic inputs: H and y within relative Frobenius error
    1e-3 of the oracle's chain (G and U differ from the exact rounding only
    where the binary32 accumulation crosses a bf16 midpoint); per element, H
    within the bound that G's and U's GEMM bounds imply through the SwiGLU
    (gpu_helpers.swiglu_bound), and y within the GEMM bound against the
    oracle's down product of the H the kernel wrote (quantized by the oracle
    with the kernel's alpha_h);
  * the chain equals the composition of the public calls bit for bit;
  * the Qwen3-8B-shaped MLP at 8192 tokens on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import (bf16_bits_to_f64, bits, check_elementwise, check_gemm_elementwise, dev,
                               gemm_bound_terms, rel_frobenius, swiglu_bound)

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _upload(codes_np, logical_scales, K, alpha):
    rows = codes_np.shape[0]
    q = mq.QuantizedTensor(rows, K, dev())
    q.codes.copy_(torch.from_numpy(np.ascontiguousarray(codes_np).reshape(-1)))
    q.scales.copy_(torch.from_numpy(oracle.scales_to_stored(logical_scales, K)))
    q.alpha.fill_(alpha)
    return q


def _swiglu_gemm(qa, qb, M, inter, K):
    h = torch.empty(M, inter, dtype=torch.bfloat16, device=dev())
    amax = torch.zeros(1, dtype=torch.float32, device=dev())
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    mq.mq_nvfp4_gemm_swiglu(qa.codes, qa.scales, qa.alpha, qb.codes, qb.scales, qb.alpha, M, inter, K, h, amax, ws)
    torch.cuda.synchronize()
    assert mq.mq_read_status(ws) == mq.MQ_OK
    return h, float(amax.item())


@pytest.mark.parametrize("M,inter,K", [(128, 128, 64), (256, 256, 256), (300, 384, 320), (1, 128, 64),
                                       (513, 256, 128), (2048, 512, 512)])
def test_swiglu_gemm_bit_exact(M, inter, K):
    """Random codes, scales 2^-2..2^2, alpha = 1: every gate and up product is
    exact in binary32, so G, U are the oracle's and H and max|h| must match."""
    rng = np.random.default_rng(M + 3 * inter + K)
    pow2 = np.array([(e + 7) << 3 for e in range(-2, 3)], np.uint8)
    ac = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    bc = rng.integers(0, 256, size=(2 * inter, K // 2), dtype=np.uint8)
    asc = pow2[rng.integers(0, 5, size=(M, K // 16))]
    bsc = pow2[rng.integers(0, 5, size=(2 * inter, K // 16))]
    h, amax = _swiglu_gemm(_upload(ac, asc, K, 1.0), _upload(bc, bsc, K, 1.0), M, inter, K)
    ref, g, u = oracle.gate_up_swiglu(ac, asc, 1.0, bc, bsc, 1.0, inter)
    got = bits(h)
    bad = np.argwhere(got != ref)
    assert len(bad) == 0, f"{len(bad)} mismatches, first {bad[:4].tolist()}"
    assert amax == float(np.max(np.abs(bf16_bits_to_f64(ref))))
    # H's NVFP4 form with its own tensor scale (R13), bit for bit
    ah = oracle.tensor_scale(ref)
    alpha = torch.empty(1, dtype=torch.float32, device=dev())
    mq.mq_alpha_from_amax(torch.tensor([amax], dtype=torch.float32, device=dev()), alpha)
    assert float(alpha.item()) == ah
    q = mq.QuantizedTensor(M, inter, dev())
    mq.mq_nvfp4_quantize(h, alpha, q.codes, q.scales)
    torch.cuda.synchronize()
    hc, hs = oracle.quantize(ref, ah)
    assert np.array_equal(q.codes.cpu().numpy().reshape(M, inter // 2), hc)
    assert np.array_equal(oracle.scales_from_stored(q.scales.cpu().numpy(), M, inter), hs)


def test_swiglu_gemm_extreme_gate_values():
    """Gate products far outside the exponential's range (|g| > 88) and exactly
    zero: silu is g, -0 or 0 there; the signs of zero come out as the oracle's."""
    M, inter, K = 128, 128, 64
    # A rows: +12 (first half), -12 (second half), 0 (first 8); gate rows 6 (scale
    # 1, or 2^-6 for half the columns), up rows 1: G = +-4608, +-72 or 0, U = +-768 or 0
    e4m3 = lambda e: (e + 7) << 3
    ac = np.full((M, K // 2), 0x77, np.uint8)                       # +6, +6
    ac[M // 2:] = 0xFF                                              # -6, -6
    ac[:8] = 0x00                                                   # zero rows
    asc = np.full((M, K // 16), e4m3(1), np.uint8)
    bc = np.full((2 * inter, K // 2), 0x77, np.uint8)
    bc[inter:] = 0x22                                               # up: +1, +1
    bsc = np.full((2 * inter, K // 16), e4m3(0), np.uint8)
    bsc[:inter // 2] = 0x08                                         # 2^-6: gate products +-72 for half the columns
    h, amax = _swiglu_gemm(_upload(ac, asc, K, 1.0), _upload(bc, bsc, K, 1.0), M, inter, K)
    ref, g, u = oracle.gate_up_swiglu(ac, asc, 1.0, bc, bsc, 1.0, inter)
    assert np.abs(bf16_bits_to_f64(g)).max() > 88.0 and (g == 0).any()
    assert np.array_equal(bits(h), ref)
    assert amax == float(np.max(np.abs(bf16_bits_to_f64(ref))))


def _check_h_elementwise(h_bits, g_ref, u_ref, xb, wgub, K, inter, rows=None):
    """H per element against the oracle's: the gate and up GEMM bounds carried
    through the SwiGLU (gpu_helpers.swiglu_bound)."""
    ax, agu = oracle.tensor_scale(xb), oracle.tensor_scale(wgub)
    xr = xb if rows is None else np.ascontiguousarray(xb[rows])
    xc, xs = oracle.quantize(xr, ax)
    gc, gs = oracle.quantize(wgub, agu)
    _, _, acc = gemm_bound_terms(oracle.dequantize(xc, xs, ax), oracle.dequantize(gc, gs, agu), K)
    bound = swiglu_bound(g_ref, u_ref, acc[:, :inter], acc[:, inter:])
    h_ref = oracle.swiglu_bf16(g_ref, u_ref)
    check_elementwise(h_bits, h_ref, bound, "h")


def _mlp_case(M, K, inter, N, seed):
    x = inputs.activation_bf16(M, K, seed=seed, outlier_channels=inputs.outlier_count(K), outlier_scale=50.0,
                               device="cuda")
    wgu = inputs.weight_bf16(2 * inter, K, seed=seed + 1, device="cuda")
    wd = inputs.weight_bf16(N, inter, seed=seed + 2, device="cuda")
    return x, wgu, wd


@pytest.mark.parametrize("M,K,inter,N", [(128, 1024, 256, 128), (300, 512, 384, 200), (1, 256, 128, 64),
                                         (2048, 1024, 1024, 512)])
def test_mlp_chain_against_oracle(M, K, inter, N):
    x, wgu, wd = _mlp_case(M, K, inter, N, seed=M + K)
    mlp = mq.MLPW4A4(wgu, wd)
    y = mlp(x)
    torch.cuda.synchronize()
    assert mq.mq_read_status(mlp._ws) == mq.MQ_OK
    ref = oracle.mlp_w4a4(bits(x), bits(wgu), bits(wd))
    # weights: same quantization as the oracle's
    assert float(mlp.wgu.alpha.item()) == oracle.tensor_scale(bits(wgu))
    h = bits(mlp.h_view(M))
    assert rel_frobenius(bf16_bits_to_f64(h), bf16_bits_to_f64(ref["h"])) <= TOL
    _check_h_elementwise(h, ref["g"], ref["u"], bits(x), bits(wgu), K, inter)
    ah = float(mlp._ws[4 * 6:4 * 7].view(torch.float32).item())      # alpha_h word of the workspace header
    assert abs(ah - ref["alpha_h"]) <= ref["alpha_h"] * 2.0 ** -7      # one bf16 step of max|h| at most
    assert rel_frobenius(bf16_bits_to_f64(bits(y)), bf16_bits_to_f64(ref["y_bf16"])) <= TOL
    # y per element: the down GEMM on the kernel's own H (alpha_h = max|h| / 2688 of that H)
    assert ah == oracle.tensor_scale(h)
    hc, hs = oracle.quantize(h, ah)
    ad = oracle.tensor_scale(bits(wd))
    dc, ds = oracle.quantize(bits(wd), ad)
    check_gemm_elementwise(bits(y), oracle.dequantize(hc, hs, ah), oracle.dequantize(dc, ds, ad), inter)
    # the running max was handed on and cleared
    assert int(mlp._ws[4 * 5:4 * 6].view(torch.int32).item()) == 0


def test_mlp_chain_equals_the_public_calls():
    """mq_mlp_w4a4 is the composition of the public entry points, bit for bit,
    and repeated calls on one workspace give identical results."""
    M, K, inter, N = 640, 1024, 512, 384
    x, wgu, wd = _mlp_case(M, K, inter, N, seed=77)
    mlp = mq.MLPW4A4(wgu, wd)
    y1 = mlp(x).clone()
    y2 = mlp(x)
    qx = mq.quantize(x)
    h, amax = _swiglu_gemm(qx, mlp.wgu, M, inter, K)
    alpha = torch.empty(1, dtype=torch.float32, device=dev())
    mq.mq_alpha_from_amax(torch.tensor([amax], dtype=torch.float32, device=dev()), alpha)
    qh = mq.QuantizedTensor(M, inter, dev())
    mq.mq_nvfp4_quantize(h, alpha, qh.codes, qh.scales)
    y3 = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
    mq.mq_nvfp4_gemm(qh.codes, qh.scales, alpha, mlp.wd.codes, mlp.wd.scales, mlp.wd.alpha, M, N, inter, y3)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y1), bits(y2))
    assert np.array_equal(bits(y1), bits(y3))
    assert np.array_equal(bits(mlp.h_view(M)), bits(h))


@pytest.mark.slow
def test_qwen3_8b_mlp_8192_tokens_sampled_rows():
    """The Qwen3-8B-shaped MLP (K 4096, inter 12288, N 4096) at 8192 tokens.
    The oracle computes the whole H in row chunks (for alpha_h, which depends
    on every element), then H and y on sampled rows are compared; alpha_h must
    agree within one bf16 step of max|h|, and equal max|h| / 2688 of the H the
    kernel wrote."""
    M, K, inter, N = 8192, 4096, 12288, 4096
    x, wgu, wd = _mlp_case(M, K, inter, N, seed=11)
    mlp = mq.MLPW4A4(wgu, wd)
    y = mlp(x)
    torch.cuda.synchronize()
    assert mq.mq_read_status(mlp._ws) == mq.MQ_OK
    xb = bits(x)
    ax = oracle.tensor_scale(xb)
    assert float(mlp._ws[12:16].view(torch.float32).item()) == ax
    xc, xs = oracle.quantize(xb, ax)
    agu = oracle.tensor_scale(bits(wgu))
    gc, gs = oracle.quantize(bits(wgu), agu)
    wgu_hat = oracle.dequantize(gc, gs, agu)
    rows = np.unique(np.concatenate([np.random.default_rng(5).choice(M, 32, replace=False), [0, M - 1]]))
    hmax_ref = 0.0
    h_ref_rows = np.empty((len(rows), inter), np.uint16)
    g_rows = np.empty((len(rows), inter), np.uint16)
    u_rows = np.empty((len(rows), inter), np.uint16)
    for r0 in range(0, M, 1024):
        y64 = oracle.gemm_f64(oracle.dequantize(xc[r0:r0 + 1024], xs[r0:r0 + 1024], ax), wgu_hat)
        g_, u_ = oracle.bf16_rne_array(y64[:, :inter]), oracle.bf16_rne_array(y64[:, inter:])
        hc_ = oracle.swiglu_bf16(g_, u_)
        hmax_ref = max(hmax_ref, float(np.max(np.abs(bf16_bits_to_f64(hc_)))))
        sel = (rows >= r0) & (rows < r0 + 1024)
        h_ref_rows[sel] = hc_[rows[sel] - r0]
        g_rows[sel] = g_[rows[sel] - r0]
        u_rows[sel] = u_[rows[sel] - r0]
    ah_ref = float(np.float32(np.float32(hmax_ref) / np.float32(2688.0)))
    h_all = mlp.h_view(M)
    h_rows = bits(h_all[torch.from_numpy(rows).to(dev())])
    assert rel_frobenius(bf16_bits_to_f64(h_rows), bf16_bits_to_f64(h_ref_rows)) <= TOL
    _check_h_elementwise(h_rows, g_rows, u_rows, xb, bits(wgu), K, inter, rows)
    ah = float(mlp._ws[24:28].view(torch.float32).item())
    assert abs(ah - ah_ref) <= ah_ref * 2.0 ** -7
    assert ah == float(np.float32(np.float32(float(h_all.abs().max().float().item())) / np.float32(2688.0)))
    ad = oracle.tensor_scale(bits(wd))
    dc, ds = oracle.quantize(bits(wd), ad)
    hc, hs = oracle.quantize(h_ref_rows, ah_ref)
    y_ref = oracle.bf16_rne_array(oracle.gemm_f64(oracle.dequantize(hc, hs, ah_ref), oracle.dequantize(dc, ds, ad)))
    y_rows = bits(y[torch.from_numpy(rows).to(dev())])
    assert rel_frobenius(bf16_bits_to_f64(y_rows), bf16_bits_to_f64(y_ref)) <= TOL
    # y per element: the down GEMM on the kernel's own H rows, quantized with the kernel's alpha_h
    hk_c, hk_s = oracle.quantize(h_rows, ah)
    check_gemm_elementwise(y_rows, oracle.dequantize(hk_c, hk_s, ah), oracle.dequantize(dc, ds, ad), inter)
