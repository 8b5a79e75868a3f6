"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
(binding in nvfp4_w4a4_quantized_03_b200.mq) and bring results back to numpy,
and the per-element error bound every random-data output comparison applies
beside the relative Frobenius error."""
import numpy as np
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import mq


def dev():
    return torch.device("cuda:0")


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def gpu_quantize(x_cpu: torch.Tensor, alpha: float | None = None):
    """alpha (from mq_tensor_scale unless given), codes [rows, K/2], stored scales."""
    rows, K = x_cpu.shape
    x = x_cpu.to(dev())
    q = mq.QuantizedTensor(rows, K, dev())
    q.scales.fill_(0xAB)   # the quantizer must overwrite padding too
    if alpha is None:
        ws = mq.workspace(mq.mq_workspace_bytes(), dev())
        mq.mq_tensor_scale(x, q.alpha, ws)
    else:
        q.alpha.fill_(alpha)
    mq.mq_nvfp4_quantize(x, q.alpha, q.codes, q.scales)
    torch.cuda.synchronize()
    return (float(q.alpha.item()), q.codes.cpu().numpy().reshape(rows, K // 2), q.scales.cpu().numpy(), q)


def rel_frobenius(y: np.ndarray, ref: np.ndarray) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(y - ref) / den) if den > 0 else float(np.linalg.norm(y))


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# -- per-element bound ------------------------------------------------------
#
# The GPU computes y = bf16(fl32(fl32(alpha_a alpha_b) * acc)), acc the fp32
# tensor-core sum of the K products p_k = (sigma q)_a (sigma q)_b, each exact in
# binary32 (at most 6 x 6 significant bits).  Whatever the order of the
# additions, and whether each one rounds to nearest or truncates, every step
# has a relative error below u = 2^-23, so |acc - sum p| <= gamma_K sum |p|
# with gamma_K = K u / (1 - K u) (Higham, Accuracy and Stability of Numerical
# Algorithms, 2nd ed., Lemma 3.1 / Section 4.2).  The two binary32 products
# add at most 2^-23 |Y|, and the oracle's binary64 sum (products rounded to
# 53 bits) less than 2^-40 S.  With Y64 = alpha sum p and S = alpha sum |p|:
#   |y - ref| <= ulp_bf16(max(|y|, |ref|)) + (gamma_K + 2^-21) S
# where the ulp term covers the two bf16 roundings (half an ulp each, of y and
# of ref) and 2^-21 S >= 2^-23 |Y| + 2^-40 S + the cross terms.

U_F32 = 2.0 ** -23


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (8 significant bits; subnormal spacing 2^-133)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7.0)


def gemm_bound_terms(a_hat: np.ndarray, w_hat: np.ndarray, K: int):
    """(reference Y64, S = sum_k |a_hat_k w_hat_k|, the accumulation part of the
    bound (gamma_K + 2^-21) S) for the rows of a_hat against all rows of w_hat."""
    y64 = oracle.gemm_f64(a_hat, w_hat)
    s = oracle.gemm_f64(np.abs(a_hat), np.abs(w_hat))
    gamma = K * U_F32 / (1.0 - K * U_F32)
    return y64, s, (gamma + 2.0 ** -21) * s


def check_elementwise(got_bits: np.ndarray, ref_bits: np.ndarray, acc_bound: np.ndarray, what: str = "y"):
    """Assert |y - ref| <= ulp_bf16(max(|y|, |ref|)) + acc_bound on every
    element (acc_bound from gemm_bound_terms); return statistics with the
    worst element (largest error / bound) for the test log."""
    y = bf16_bits_to_f64(got_bits)
    r = bf16_bits_to_f64(ref_bits)
    assert y.shape == r.shape == acc_bound.shape, (y.shape, r.shape, acc_bound.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - r)
    bound = bf16_ulp(np.maximum(np.abs(y), np.abs(r))) + acc_bound
    ratio = err / bound
    i = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
    ulps = err / bf16_ulp(r)
    stats = dict(what=what, worst_ratio=float(ratio[i]), worst_index=tuple(int(v) for v in i),
                 worst_y=float(y[i]), worst_ref=float(r[i]), worst_bound=float(bound[i]),
                 max_err_ulps=float(ulps.max()), frac_differ=float(np.mean(err > 0)),
                 frac_over_1ulp=float(np.mean(ulps > 1.0)))
    print(stats)
    assert ratio[i] <= 1.0, stats
    return stats


def check_gemm_elementwise(got_bits: np.ndarray, a_hat: np.ndarray, w_hat: np.ndarray, K: int, what: str = "y"):
    """Per-element bound of a GEMM output against the oracle on the same
    quantized operands, plus the relative Frobenius error; returns (stats, err)."""
    y64, _, accb = gemm_bound_terms(a_hat, w_hat, K)
    ref = oracle.bf16_rne_array(y64)
    stats = check_elementwise(got_bits, ref, accb, what)
    return stats, rel_frobenius(bf16_bits_to_f64(got_bits), bf16_bits_to_f64(ref))


def swiglu_bound(g_ref: np.ndarray, u_ref: np.ndarray, g_acc: np.ndarray, u_acc: np.ndarray) -> np.ndarray:
    """Bound on |h_gpu - h_ref| beyond the bf16 rounding of h, where h =
    bf16(silu(G) U) and the GPU's G and U (bf16 GEMM outputs) are within
    e = ulp_bf16(.) + acc of the oracle's g_ref, u_ref (gemm_bound_terms).
    Both sides run the same binary32 SwiGLU, so the difference comes from the
    inputs: |d silu/dg| <= 1.1 and |silu(g)| <= |g|, giving
      |dh| <= 1.1 (|u| + e_u) e_g + (|g| + 1.1 e_g) e_u + 2^-20 |h|-scale terms."""
    g = bf16_bits_to_f64(g_ref)
    u = bf16_bits_to_f64(u_ref)
    eg = 2.0 * bf16_ulp(np.abs(g) + g_acc) + g_acc
    eu = 2.0 * bf16_ulp(np.abs(u) + u_acc) + u_acc
    return 1.1 * (np.abs(u) + eu) * eg + (np.abs(g) + 1.1 * eg) * eu + 2.0 ** -20 * (np.abs(g) + eg) * (np.abs(u) + eu)


# -- the quantized activation mq_linear_w4a4 leaves in its workspace ---------
#
# Workspace layout of mq_linear_w4a4 (library-internal, fixed by
# csrc/mq_api.cu): a 256-byte header, the readiness flags of the fused form
# (one int per 128-row block and 256-element K stage, rounded up to 256
# bytes), the codes of X (rounded up to 256 bytes), then the scales of X.

def _round256(v: int) -> int:
    return (v + 255) // 256 * 256


def linear_ws_offsets(M: int, K: int):
    flags = (M + 127) // 128 * ((K // 64 + 3) // 4)
    codes_off = 256 + _round256(4 * flags)
    scales_off = codes_off + _round256(M * K // 2)
    return codes_off, scales_off


def linear_ws_codes_rows(ws: torch.Tensor, M: int, K: int, rows: np.ndarray | None = None) -> np.ndarray:
    """The linear's codes of X (rows given, or all) as uint8 [rows, K/2]."""
    off, _ = linear_ws_offsets(M, K)
    codes = ws[off:off + M * K // 2].view(M, K // 2)
    if rows is not None:
        codes = codes[torch.from_numpy(np.asarray(rows, np.int64)).to(ws.device)]
    return codes.cpu().numpy()


def linear_ws_scales(ws: torch.Tensor, M: int, K: int) -> np.ndarray:
    """The linear's stored scales of X (MMA order, padded rows included)."""
    _, off = linear_ws_offsets(M, K)
    return ws[off:off + mq.mq_nvfp4_scales_bytes(M, K)].cpu().numpy()
