"""Failure detection without a fault: a GEMM whose pipeline is starved on
purpose (mq_debug_gemm_stall withholds the first stage's loads and shortens
every bounded wait) must end by itself with MQ_ERR_TIMEOUT in the workspace
status word, and the CUDA context must stay usable for the next call."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import bf16_bits_to_f64, bits, dev, rel_frobenius

pytestmark = pytest.mark.gpu


def _stall_fn():
    f = mq.lib().mq_debug_gemm_stall
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, ctypes.c_size_t, i64, vp]
    f.restype = ctypes.c_int
    return f


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("form", ["1", "2"])
def test_stalled_gemm_reports_timeout_and_context_survives(form, switches):
    switches(gemm_form=int(form))
    M, N, K = 256, 512, 1024
    x = inputs.activation_bf16(M, K, seed=9, outlier_channels=10).to(dev())
    w = inputs.weight_bf16(N, K, seed=10).to(dev())
    qx, qw = mq.quantize(x), mq.quantize(w)
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.time()
    st = _stall_fn()(_p(qx.codes), _p(qx.scales), _p(qx.alpha), _p(qw.codes), _p(qw.scales), _p(qw.alpha),
                     M, N, K, _p(y), _p(ws), ws.numel(), 2_000_000, stream)
    assert st == mq.MQ_OK
    torch.cuda.synchronize()
    assert time.time() - t0 < 30.0
    assert mq.mq_read_status(ws) == mq.MQ_ERR_TIMEOUT
    assert mq.mq_read_status(ws) == mq.MQ_OK          # reading clears the word

    # the same context, stream and workspace keep working
    mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, qw.codes, qw.scales, qw.alpha, M, N, K, y, ws)
    torch.cuda.synchronize()
    assert mq.mq_read_status(ws) == mq.MQ_OK
    ref = oracle.linear_w4a4(bits(x.cpu()), bits(w.cpu()))
    assert rel_frobenius(bf16_bits_to_f64(bits(y)), bf16_bits_to_f64(ref["y_bf16"])) <= 1e-3


def test_stalled_decode_gemm_reports_timeout_and_context_survives():
    """The decode form (M <= 64, split-K over a cluster): every CTA withholds
    its first stage, all bounded waits run out, the copies already issued land
    before the CTAs end, and the next decode GEMM is correct."""
    M, N, K = 8, 1024, 4096
    x = inputs.activation_bf16(M, K, seed=19, outlier_channels=10).to(dev())
    w = inputs.weight_bf16(N, K, seed=20).to(dev())
    qx, qw = mq.quantize(x), mq.quantize(w)
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _stall_fn()(_p(qx.codes), _p(qx.scales), _p(qx.alpha), _p(qw.codes), _p(qw.scales), _p(qw.alpha),
                     M, N, K, _p(y), _p(ws), ws.numel(), 2_000_000, stream)
    assert st == mq.MQ_OK
    torch.cuda.synchronize()
    assert mq.mq_read_status(ws) == mq.MQ_ERR_TIMEOUT
    mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, qw.codes, qw.scales, qw.alpha, M, N, K, y, ws)
    torch.cuda.synchronize()
    assert mq.mq_read_status(ws) == mq.MQ_OK
    ref = oracle.linear_w4a4(bits(x.cpu()), bits(w.cpu()))
    assert rel_frobenius(bf16_bits_to_f64(bits(y)), bf16_bits_to_f64(ref["y_bf16"])) <= 1e-3


def test_stall_hook_validates_its_limit():
    f = _stall_fn()
    dummy = ctypes.c_void_p(1 << 20)
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    assert f(dummy, dummy, dummy, dummy, dummy, dummy, 128, 256, 64, dummy, _p(ws), ws.numel(), 10, None) == -1
