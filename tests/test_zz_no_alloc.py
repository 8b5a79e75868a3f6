"""The allocation-free linear entry point (mq_linear_w4a4_noalloc).

It serves callers that cannot allocate device memory -- a plugin inside an
application that owns all device memory and offers extensions no allocator,
or C code that must not call cudaMalloc because it synchronizes the device.
It runs the same kernels as mq_linear_w4a4 with the library's own static
scratch in place of a caller workspace, so its output must match
mq_linear_w4a4 on the same inputs.  This file is collected last so that a run
stopping at the first failure has already run every other test; it passes
alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import bf16_bits_to_f64, bits, dev, rel_frobenius

pytestmark = pytest.mark.gpu
TOL = 1e-3   # the tolerance the GEMM parity tests use


def _noalloc_fn():
    f = mq.lib().mq_linear_w4a4_noalloc
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp]
    f.restype = ctypes.c_int
    return f


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    K, N = 1024, 768
    w = inputs.weight_bf16(N, K, seed=21).to(dev())
    qw = mq.quantize(w)
    # two calls in a row, different activations (different alpha_x and M)
    for call, (M, seed, scale) in enumerate([(200, 1, 50.0), (131, 2, 5.0)]):
        x = inputs.activation_bf16(M, K, seed=seed, outlier_channels=10, outlier_scale=scale).to(dev())
        y_ref = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
        ws = mq.workspace(mq.mq_linear_w4a4_workspace_bytes(M, K), dev())
        mq.mq_linear_w4a4(x, qw.codes, qw.scales, qw.alpha, N, y_ref, ws)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev())
        st = f(_p(x), M, K, _p(qw.codes), _p(qw.scales), _p(qw.alpha), N, _p(y), stream)
        assert st == 0, mq.lib().mq_status_string(st)
        torch.cuda.synchronize()
        got, ref = bits(y), bits(y_ref)
        err = rel_frobenius(bf16_bits_to_f64(got), bf16_bits_to_f64(ref))
        assert err <= TOL, (call, err)
        assert np.array_equal(got, ref), f"call {call}: outputs differ"


def test_noalloc_refuses_shapes_beyond_its_scratch():
    f = _noalloc_fn()
    M, K, N = 131072, 4096, 4096
    assert mq.mq_linear_w4a4_workspace_bytes(M, K) > mq.MQ_NOALLOC_SCRATCH_BYTES
    dummy = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: the size check comes first
    st = f(dummy, M, K, dummy, dummy, dummy, N, dummy, None)
    assert st == -5, mq.lib().mq_status_string(st)      # MQ_ERR_WORKSPACE


def test_noalloc_after_a_call_that_left_its_header_dirty():
    """A call ended by a timeout can leave the scratch header's ticket, running
    max, generation and status words nonzero; the next call clears the header
    before its kernels run, so its output is the workspace entry point's."""
    f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    M, K, N = 300, 2048, 512
    w = inputs.weight_bf16(N, K, seed=23).to(dev())
    qw = mq.quantize(w)
    x = inputs.activation_bf16(M, K, seed=24, outlier_channels=20, outlier_scale=30.0).to(dev())
    y_ref = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
    ws = mq.workspace(mq.mq_linear_w4a4_workspace_bytes(M, K), dev())
    mq.mq_linear_w4a4(x, qw.codes, qw.scales, qw.alpha, N, y_ref, ws)
    for word in (0xFFFFFFFF, 0x00000001, 0x7F7F0003):
        assert mq.lib().mq_debug_noalloc_fill_header(word, stream) == 0
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev())
        st = f(_p(x), M, K, _p(qw.codes), _p(qw.scales), _p(qw.alpha), N, _p(y), stream)
        assert st == 0, mq.lib().mq_status_string(st)
        torch.cuda.synchronize()
        assert np.array_equal(bits(y), bits(y_ref)), hex(word)
