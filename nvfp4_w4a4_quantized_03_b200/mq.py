"""ctypes binding of libmq.so (C ABI in include/mq.h).

Argument marshalling only: every step of the quantizer and the GEMM runs in
the CUDA kernels of libmq.so.  There is no CPU fallback; if the library has
not been built or the current device is not a B200 (sm_100a), calls raise.

The functions keep the C names.  They take torch CUDA tensors (for device
memory) and enqueue on the current torch stream unless `stream` is given.
With MQ_DEBUG=1 in the environment the debug build (libmq_debug.so, every
index-computed access and TMA coordinate bounds-checked) is loaded instead.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmq_debug.so" if os.environ.get("MQ_DEBUG") == "1" else "libmq.so")

MQ_OK = 0
MQ_ERR_TIMEOUT = -7

_lib = None


class MQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().mq_status_string(status).decode()} ({status})")


def lib() -> ctypes.CDLL:
    """Load libmq.so (built by ``python -m nvfp4_w4a4_quantized_03_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m nvfp4_w4a4_quantized_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        L.mq_status_string.argtypes = [ctypes.c_int]
        L.mq_status_string.restype = ctypes.c_char_p
        for name in ("mq_nvfp4_codes_bytes", "mq_nvfp4_scales_bytes", "mq_linear_w4a4_workspace_bytes"):
            getattr(L, name).argtypes = [i64, i64]
            getattr(L, name).restype = sz
        L.mq_workspace_bytes.argtypes = []
        L.mq_workspace_bytes.restype = sz
        L.mq_tensor_scale.argtypes = [vp, i64, vp, vp, sz, vp]
        L.mq_tensor_amax.argtypes = [vp, i64, vp, vp, sz, vp]
        L.mq_alpha_from_amax.argtypes = [vp, vp, vp]
        L.mq_nvfp4_quantize.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.mq_nvfp4_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]
        L.mq_linear_w4a4.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp, sz, vp]
        L.mq_read_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
        L.mq_nvfp4_gemm_swiglu.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, sz, vp]
        L.mq_mlp_w4a4_workspace_bytes.argtypes = [i64, i64, i64]
        L.mq_mlp_w4a4_workspace_bytes.restype = sz
        L.mq_mlp_w4a4.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp, vp, i64, vp, vp, sz, vp]
        L.mq_is_debug_build.argtypes = []
        L.mq_debug_bounds_hits.argtypes = [ctypes.POINTER(ctypes.c_int64)]
        L.mq_set_switch.argtypes = [ctypes.c_int, ctypes.c_int]
        L.mq_get_switch.argtypes = [ctypes.c_int]
        L.mq_debug_noalloc_fill_header.argtypes = [ctypes.c_uint32, vp]
        for name in ("mq_tensor_scale", "mq_tensor_amax", "mq_alpha_from_amax", "mq_nvfp4_quantize",
                     "mq_nvfp4_gemm", "mq_linear_w4a4", "mq_read_status", "mq_nvfp4_gemm_swiglu",
                     "mq_mlp_w4a4", "mq_is_debug_build", "mq_debug_bounds_hits", "mq_set_switch",
                     "mq_get_switch", "mq_debug_noalloc_fill_header"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, what: str):
    if status != MQ_OK:
        raise MQError(status, what)


# -- selectable alternatives (MQ_SWITCH_* in mq.h) -------------------------

SWITCHES = {"linear_path": 0, "gemm_form": 1, "gemm_decode": 2, "decode_split": 3, "gemm_stages": 4,
            "gemm_group_m": 5, "pdl": 6}
LINEAR_PATHS = {"onepass": 0, "split": 1, "ingemm": 2}


def _switch_id(name) -> int:
    return name if isinstance(name, int) else SWITCHES[name]


def mq_set_switch(name, value: int) -> None:
    """Set a process-wide switch by name (SWITCHES) or MQ_SWITCH_* number;
    the linear path also takes its name (LINEAR_PATHS)."""
    if name == "linear_path" and isinstance(value, str):
        value = LINEAR_PATHS[value]
    _check(lib().mq_set_switch(_switch_id(name), int(value)), f"mq_set_switch({name}, {value})")


def mq_get_switch(name) -> int:
    v = int(lib().mq_get_switch(_switch_id(name)))
    if v < 0:
        raise MQError(v, f"mq_get_switch({name})")
    return v


class switch:
    """Context manager: `with mq.switch(gemm_form=2): ...` sets switches for
    the block and puts the previous values back afterwards."""

    def __init__(self, **values):
        self.values = values
        self.saved = {}

    def __enter__(self):
        for name, v in self.values.items():
            self.saved[name] = mq_get_switch(name)
            mq_set_switch(name, v)
        return self

    def __exit__(self, *exc):
        for name, v in self.saved.items():
            mq_set_switch(name, v)
        return False


# -- sizes ------------------------------------------------------------------

def mq_nvfp4_codes_bytes(rows: int, K: int) -> int:
    return int(lib().mq_nvfp4_codes_bytes(rows, K))


def mq_nvfp4_scales_bytes(rows: int, K: int) -> int:
    return int(lib().mq_nvfp4_scales_bytes(rows, K))


def mq_workspace_bytes() -> int:
    return int(lib().mq_workspace_bytes())


def mq_linear_w4a4_workspace_bytes(M: int, K: int) -> int:
    return int(lib().mq_linear_w4a4_workspace_bytes(M, K))


# -- calls ------------------------------------------------------------------

def mq_tensor_scale(x: torch.Tensor, alpha: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    assert x.dtype == torch.bfloat16 and alpha.dtype == torch.float32
    _check(lib().mq_tensor_scale(_ptr(x), x.numel(), _ptr(alpha), _ptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream)), "mq_tensor_scale")


def mq_tensor_amax(x: torch.Tensor, amax: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    assert x.dtype == torch.bfloat16 and amax.dtype == torch.float32
    _check(lib().mq_tensor_amax(_ptr(x), x.numel(), _ptr(amax), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)), "mq_tensor_amax")


def mq_alpha_from_amax(amax: torch.Tensor, alpha: torch.Tensor, stream=None) -> None:
    assert amax.dtype == torch.float32 and alpha.dtype == torch.float32
    _check(lib().mq_alpha_from_amax(_ptr(amax), _ptr(alpha), _stream(stream)), "mq_alpha_from_amax")


def mq_nvfp4_quantize(x: torch.Tensor, alpha: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                      stream=None) -> None:
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    rows, K = x.shape
    assert codes.numel() * codes.element_size() >= mq_nvfp4_codes_bytes(rows, K)
    assert scales.numel() * scales.element_size() >= mq_nvfp4_scales_bytes(rows, K)
    _check(lib().mq_nvfp4_quantize(_ptr(x), rows, K, _ptr(alpha), _ptr(codes), _ptr(scales), _stream(stream)),
           "mq_nvfp4_quantize")


def mq_nvfp4_gemm(a_codes, a_scales, alpha_a, b_codes, b_scales, alpha_b, M: int, N: int, K: int,
                  y: torch.Tensor, ws: torch.Tensor | None = None, stream=None) -> None:
    assert y.dtype == torch.bfloat16 and y.numel() >= M * N
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().mq_nvfp4_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(alpha_a), _ptr(b_codes), _ptr(b_scales),
                               _ptr(alpha_b), M, N, K, _ptr(y), _ptr(ws), ws_bytes, _stream(stream)),
           "mq_nvfp4_gemm")


def mq_linear_w4a4(x: torch.Tensor, w_codes, w_scales, alpha_w, N: int, y: torch.Tensor, ws: torch.Tensor,
                   stream=None) -> None:
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and y.dtype == torch.bfloat16
    M, K = x.shape
    _check(lib().mq_linear_w4a4(_ptr(x), M, K, _ptr(w_codes), _ptr(w_scales), _ptr(alpha_w), N, _ptr(y),
                                _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "mq_linear_w4a4")


def mq_nvfp4_gemm_swiglu(a_codes, a_scales, alpha_a, b_codes, b_scales, alpha_b, M: int, inter: int, K: int,
                         h: torch.Tensor, h_amax: torch.Tensor, ws: torch.Tensor | None = None, stream=None) -> None:
    assert h.dtype == torch.bfloat16 and h.numel() >= M * inter and h_amax.dtype == torch.float32
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().mq_nvfp4_gemm_swiglu(_ptr(a_codes), _ptr(a_scales), _ptr(alpha_a), _ptr(b_codes), _ptr(b_scales),
                                      _ptr(alpha_b), M, inter, K, _ptr(h), _ptr(h_amax), _ptr(ws), ws_bytes,
                                      _stream(stream)), "mq_nvfp4_gemm_swiglu")


def mq_mlp_w4a4_workspace_bytes(M: int, K: int, inter: int) -> int:
    return int(lib().mq_mlp_w4a4_workspace_bytes(M, K, inter))


def mq_mlp_w4a4(x: torch.Tensor, wgu_codes, wgu_scales, alpha_gu, inter: int, wd_codes, wd_scales, alpha_d,
                N: int, y: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and y.dtype == torch.bfloat16
    M, K = x.shape
    _check(lib().mq_mlp_w4a4(_ptr(x), M, K, _ptr(wgu_codes), _ptr(wgu_scales), _ptr(alpha_gu), inter,
                             _ptr(wd_codes), _ptr(wd_scales), _ptr(alpha_d), N, _ptr(y), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "mq_mlp_w4a4")


def mq_is_debug_build() -> bool:
    return bool(lib().mq_is_debug_build())


def mq_debug_bounds_hits() -> int:
    """Failed bounds checks since the previous call (synchronizes the device;
    always 0 in the release build)."""
    out = ctypes.c_int64(0)
    _check(lib().mq_debug_bounds_hits(ctypes.byref(out)), "mq_debug_bounds_hits")
    return int(out.value)


def mq_read_status(ws: torch.Tensor, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(lib().mq_read_status(_ptr(ws), _stream(stream), ctypes.byref(out)), "mq_read_status")
    return int(out.value)


# -- conveniences (allocation through torch, then the calls above) ----------

class QuantizedTensor:
    """NVFP4 tensor [rows, K]: packed codes, MMA-ordered scales, alpha (device)."""

    def __init__(self, rows: int, K: int, device):
        self.rows, self.K = rows, K
        self.codes = torch.empty(mq_nvfp4_codes_bytes(rows, K), dtype=torch.uint8, device=device)
        self.scales = torch.empty(mq_nvfp4_scales_bytes(rows, K), dtype=torch.uint8, device=device)
        self.alpha = torch.empty(1, dtype=torch.float32, device=device)


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled workspace buffer (the calls keep its counters at zero)."""
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def quantize(x: torch.Tensor, ws: torch.Tensor | None = None, stream=None) -> QuantizedTensor:
    """alpha_x of x, then its NVFP4 codes and scales (e.g. offline weight quantization)."""
    rows, K = x.shape
    q = QuantizedTensor(rows, K, x.device)
    if ws is None:
        ws = workspace(mq_workspace_bytes(), x.device)
    mq_tensor_scale(x, q.alpha, ws, stream)
    mq_nvfp4_quantize(x, q.alpha, q.codes, q.scales, stream)
    return q


class LinearW4A4:
    """A linear layer y = x W^T on the FP4 prefill path: W quantized once at
    construction, x quantized per call inside mq_linear_w4a4."""

    def __init__(self, weight: torch.Tensor):
        assert weight.dtype == torch.bfloat16 and weight.is_cuda
        self.N, self.K = weight.shape
        self.w = quantize(weight.contiguous())
        self._ws = None

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        M, K = x.shape
        assert K == self.K
        need = mq_linear_w4a4_workspace_bytes(M, K)
        if self._ws is None or self._ws.numel() < need:
            self._ws = workspace(need, x.device)
        if out is None:
            out = torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
        mq_linear_w4a4(x, self.w.codes, self.w.scales, self.w.alpha, self.N, out, self._ws, stream)
        return out


class MLPW4A4:
    """A decoder MLP on the FP4 prefill path: y = (SwiGLU(x Wg^T, x Wu^T)) Wd^T
    with both linears W4A4.  The gate and up weights are quantized as one
    [2 inter, K] tensor (gate rows first), the down weight [N, inter] on its
    own, once at construction; x and H are quantized per call."""

    def __init__(self, w_gate_up: torch.Tensor, w_down: torch.Tensor):
        assert w_gate_up.dtype == torch.bfloat16 and w_down.dtype == torch.bfloat16
        two_inter, self.K = w_gate_up.shape
        self.inter = two_inter // 2
        self.N = w_down.shape[0]
        assert two_inter == 2 * self.inter and w_down.shape[1] == self.inter
        self.wgu = quantize(w_gate_up.contiguous())
        self.wd = quantize(w_down.contiguous())
        self._ws = None

    def workspace(self, M: int, device) -> torch.Tensor:
        need = mq_mlp_w4a4_workspace_bytes(M, self.K, self.inter)
        if self._ws is None or self._ws.numel() < need:
            self._ws = workspace(need, device)
        return self._ws

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        M, K = x.shape
        assert K == self.K
        ws = self.workspace(M, x.device)
        if out is None:
            out = torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
        mq_mlp_w4a4(x, self.wgu.codes, self.wgu.scales, self.wgu.alpha, self.inter, self.wd.codes, self.wd.scales,
                    self.wd.alpha, self.N, out, ws, stream)
        return out

    def h_view(self, M: int) -> torch.Tensor:
        """H [M, inter] as the last call left it in the workspace."""
        off = mq_linear_w4a4_workspace_bytes(M, self.K)
        return self._ws[off:off + M * self.inter * 2].view(torch.bfloat16).view(M, self.inter)


# -- the allocation-free variant (library-owned scratch) ---------------------

MQ_NOALLOC_SCRATCH_BYTES = 64 << 20


def mq_linear_w4a4_noalloc(x: torch.Tensor, w_codes, w_scales, alpha_w, N: int, y: torch.Tensor,
                           stream=None) -> None:
    """mq_linear_w4a4 without a workspace, for callers that cannot allocate:
    the library's static 64 MiB scratch is used (shared by every call on a
    device, so calls must not overlap on the GPU)."""
    f = lib().mq_linear_w4a4_noalloc
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp]
    f.restype = ctypes.c_int
    M, K = x.shape
    _check(f(_ptr(x), M, K, _ptr(w_codes), _ptr(w_scales), _ptr(alpha_w), N, _ptr(y), _stream(stream)),
           "mq_linear_w4a4_noalloc")
