"""Plain CPU oracle for the NVFP4 W4A4 linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may use this package; the CUDA library and its
Python binding never do.  It shares no code with the CUDA path.

The scalar work (E2M1 / E4M3 rounding, the per-block quantizer, the
dequantizer, bf16 rounding) lives in ``mq_oracle.c``; the one library primitive
used is numpy's binary64 matrix product for the contraction.

Formulas followed (NVFP4 two-level microscaling):
  "Mix-Quant：面向智能体LLM的量化预填充与精确解码" (paper.rainbus.top digest),
  section 方法步骤详情, step (3); "Mix-Quant: Quantized Prefilling, Precise
  Decoding for Agentic LLMs" (r9-hu paper digest), section Method, item 1:
    sigma_b = Pi_E4M3(max_{i in b}|x_i| / (alpha_x q_max)),
    q_i = Pi_FP4(x_i / (alpha_x sigma_b(i))),  xhat_i = alpha_x sigma_b(i) q_i,
  blocks of 16 along K, round to nearest.  The readings taken where the pages
  are silent are listed in ``mq_oracle.c`` (R1..R8 at the top, R11..R13 with
  the SwiGLU of the MLP; R9 and R10, the block axis and one alpha per fused
  weight, are how the inputs are laid out).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

GROUP = 16  # elements per block scale


def build(force: bool = False) -> str:
    """Compile mq_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_bf16_rne.argtypes = [ctypes.c_double]
        lib.oracle_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_tensor_scale.argtypes = [u16p, i64]
        lib.oracle_tensor_scale.restype = ctypes.c_float
        for name in ("oracle_quantize", "oracle_quantize_exact"):
            getattr(lib, name).argtypes = [u16p, i64, i64, ctypes.c_float, u8p, u8p]
            getattr(lib, name).restype = None
        lib.oracle_dequantize.argtypes = [u8p, u8p, i64, i64, ctypes.c_float, f64p]
        lib.oracle_dequantize.restype = None
        lib.oracle_bf16_rne_array.argtypes = [f64p, i64, u16p]
        lib.oracle_bf16_rne_array.restype = None
        lib.oracle_scale_offset.argtypes = [i64, i64, i64]
        lib.oracle_scale_offset.restype = i64
        lib.oracle_scale_bytes.argtypes = [i64, i64]
        lib.oracle_scale_bytes.restype = i64
        lib.oracle_scales_to_stored.argtypes = [u8p, i64, i64, u8p]
        lib.oracle_scales_from_stored.argtypes = [u8p, i64, i64, u8p]
        lib.oracle_exp_f32.argtypes = [ctypes.c_float]
        lib.oracle_exp_f32.restype = ctypes.c_float
        lib.oracle_silu_f32.argtypes = [ctypes.c_float]
        lib.oracle_silu_f32.restype = ctypes.c_float
        lib.oracle_swiglu_bf16.argtypes = [ctypes.c_uint16, ctypes.c_uint16]
        lib.oracle_swiglu_bf16.restype = ctypes.c_uint16
        lib.oracle_swiglu_array.argtypes = [u16p, u16p, i64, u16p]
        lib.oracle_swiglu_array.restype = None
        _lib = lib
    return _lib


def _p(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _bits(x) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 array of its bit patterns."""
    if hasattr(x, "dtype") and str(getattr(x, "dtype")) == "torch.bfloat16":
        x = x.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 bit patterns expected as uint16"
    return x


def num_threads() -> int:
    return int(_L().oracle_num_threads())


# -- scalars ----------------------------------------------------------------

def e2m1_encode(v: float) -> int:
    return int(_L().oracle_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(_L().oracle_e2m1_decode(code))


def e4m3_encode(v: float) -> int:
    return int(_L().oracle_e4m3_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return float(_L().oracle_e4m3_decode(code))


def bf16_to_f32(bits: int) -> float:
    return float(_L().oracle_bf16_to_f32(bits))


def bf16_rne(v: float) -> int:
    return int(_L().oracle_bf16_rne(float(v)))


# -- tensors ----------------------------------------------------------------

def tensor_scale(x) -> float:
    """alpha_x = fl32(max|x| / 2688) of a bf16 tensor (1.0 for an all-zero tensor)."""
    xb = _bits(x).reshape(-1)
    return float(_L().oracle_tensor_scale(_p(xb, ctypes.c_uint16), xb.size))


def quantize(x, alpha: float, exact: bool = False):
    """Quantize a bf16 [rows, K] tensor.

    Returns (codes uint8 [rows, K/2], scales uint8 [rows, K/16]) with scales in
    plain row-major order.  ``exact=True`` uses the exact-real reading of the
    two formulas instead of the block-reciprocal reading.
    """
    xb = _bits(x)
    rows, K = xb.shape
    assert K % GROUP == 0
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // GROUP), np.uint8)
    fn = _L().oracle_quantize_exact if exact else _L().oracle_quantize
    fn(_p(xb, ctypes.c_uint16), rows, K, ctypes.c_float(alpha),
       _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8))
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, alpha: float) -> np.ndarray:
    """xhat = alpha * sigma_b * q in binary64, shape [rows, K]."""
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, K), np.float64)
    _L().oracle_dequantize(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), rows, K,
                           ctypes.c_float(alpha), _p(out, ctypes.c_double))
    return out


def bf16_rne_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    _L().oracle_bf16_rne_array(_p(v, ctypes.c_double), v.size, _p(out, ctypes.c_uint16))
    return out


def gemm_f64(a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """Y64[m, n] = sum_k a_hat[m, k] * w_hat[n, k] (binary64 matrix product)."""
    return np.asarray(a_hat, np.float64) @ np.asarray(w_hat, np.float64).T


def linear_w4a4(x, w, w_quant=None):
    """End-to-end reference of the W4A4 linear: Y = bf16(xhat . what^T).

    Returns a dict with alpha_x, codes/scales of X, alpha_w, codes/scales of W,
    the binary64 product and its bf16 bit patterns.
    """
    ax = tensor_scale(x)
    xc, xs = quantize(x, ax)
    if w_quant is None:
        aw = tensor_scale(w)
        wc, ws = quantize(w, aw)
    else:
        aw, wc, ws = w_quant
    y64 = gemm_f64(dequantize(xc, xs, ax), dequantize(wc, ws, aw))
    return dict(alpha_x=ax, x_codes=xc, x_scales=xs, alpha_w=aw, w_codes=wc,
                w_scales=ws, y64=y64, y_bf16=bf16_rne_array(y64))


# -- scale storage order consumed by the block-scaled MMA -------------------

def scale_offset(row: int, kblock: int, K: int) -> int:
    return int(_L().oracle_scale_offset(row, kblock, K))


def scale_bytes(rows: int, K: int) -> int:
    return int(_L().oracle_scale_bytes(rows, K))


def scales_to_stored(logical: np.ndarray, K: int) -> np.ndarray:
    logical = np.ascontiguousarray(logical, np.uint8)
    rows = logical.shape[0]
    out = np.empty(scale_bytes(rows, K), np.uint8)
    _L().oracle_scales_to_stored(_p(logical, ctypes.c_uint8), rows, K, _p(out, ctypes.c_uint8))
    return out


def scales_from_stored(stored: np.ndarray, rows: int, K: int) -> np.ndarray:
    stored = np.ascontiguousarray(stored, np.uint8).reshape(-1)
    assert stored.size >= scale_bytes(rows, K)
    out = np.empty((rows, K // GROUP), np.uint8)
    _L().oracle_scales_from_stored(_p(stored, ctypes.c_uint8), rows, K, _p(out, ctypes.c_uint8))
    return out


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[rows, K/2] packed bytes -> [rows, K] 4-bit codes (low nibble first)."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out


# -- the MLP: gate/up linear, SwiGLU, down linear ---------------------------

def exp_f32(x: float) -> float:
    """The binary32 exponential of the SwiGLU (Cody-Waite reduction, degree-7 Taylor)."""
    return float(_L().oracle_exp_f32(float(x)))


def silu_f32(g: float) -> float:
    return float(_L().oracle_silu_f32(float(g)))


def swiglu_bf16(g, u) -> np.ndarray:
    """h = bf16(fl32(silu(g) * u)) elementwise on bf16 bit patterns."""
    gb = np.ascontiguousarray(_bits(g))
    ub = np.ascontiguousarray(_bits(u))
    assert gb.shape == ub.shape
    out = np.empty(gb.shape, np.uint16)
    _L().oracle_swiglu_array(_p(gb, ctypes.c_uint16), _p(ub, ctypes.c_uint16), gb.size,
                             _p(out, ctypes.c_uint16))
    return out


def gate_up_swiglu(x_codes, x_scales, alpha_x, wgu_codes, wgu_scales, alpha_gu, inter: int):
    """H of the MLP from quantized operands: the gate/up product of xhat with
    the [2 * inter, K] weight (gate rows first, then up rows), rounded to bf16
    as the linear writes it, then SwiGLU.  Returns (h bits [M, inter], G, U)."""
    y64 = gemm_f64(dequantize(x_codes, x_scales, alpha_x), dequantize(wgu_codes, wgu_scales, alpha_gu))
    g = bf16_rne_array(y64[:, :inter])
    u = bf16_rne_array(y64[:, inter:])
    return swiglu_bf16(g, u), g, u


def mlp_w4a4(x, wgu, wd, wgu_quant=None, wd_quant=None):
    """End-to-end reference of the W4A4 MLP: the gate/up linear (A1-A6),
    SwiGLU (R11, R12), the down linear on H quantized with its own alpha (R13).
    ``wgu`` is [2 * inter, K] with the gate rows first."""
    inter = (wgu_quant[1].shape[0] if wgu_quant is not None else _bits(wgu).shape[0]) // 2
    ax = tensor_scale(x)
    xc, xs = quantize(x, ax)
    if wgu_quant is None:
        agu = tensor_scale(wgu)
        gc, gs = quantize(wgu, agu)
    else:
        agu, gc, gs = wgu_quant
    if wd_quant is None:
        ad = tensor_scale(wd)
        dc, ds = quantize(wd, ad)
    else:
        ad, dc, ds = wd_quant
    h, g, u = gate_up_swiglu(xc, xs, ax, gc, gs, agu, inter)
    ah = tensor_scale(h)
    hc, hs = quantize(h, ah)
    y64 = gemm_f64(dequantize(hc, hs, ah), dequantize(dc, ds, ad))
    return dict(alpha_x=ax, h=h, g=g, u=u, alpha_h=ah, h_codes=hc, h_scales=hs, y64=y64,
                y_bf16=bf16_rne_array(y64))
