"""The prefill sequence of linears (nvfp4_w4a4_quantized_03_b200.sequence):
a CUDA-graph replay gives the eager result bit for bit, the shared workspace
reports no device error, and a projection of the last layer matches the
oracle on sampled rows (NVFP4 W4A4 linear, "Mix-Quant：面向智能体LLM的量化预填充
与精确解码", section 方法步骤详情, step (3)).  With the fused MLP, the last
layer's MLP output matches the oracle's MLP chain (readings R11-R13 of the
oracle for the activation between the two linears)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from nvfp4_w4a4_quantized_03_b200.sequence import PrefillSequence
from tests.gpu_helpers import bf16_bits_to_f64, bits, check_gemm_elementwise, dev, rel_frobenius

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager_and_oracle():
    seq = PrefillSequence(layers=3, tokens=640, device=dev())
    seq.run()
    torch.cuda.synchronize()
    eager = [bits(y) for y in seq.y]
    seq.capture()
    for y in seq.y:
        y.fill_(float("nan"))
    seq.replay()
    seq.replay()
    torch.cuda.synchronize()
    assert seq.status() == mq.MQ_OK
    for e, y in zip(eager, seq.y):
        assert np.array_equal(bits(y), e)
    # the last layer's gate/up projection against the oracle, 48 sampled rows
    i = [p.name for p in inputs.QWEN3_8B_PROJECTIONS].index("gate_up")
    p = inputs.QWEN3_8B_PROJECTIONS[i]
    xb = bits(seq.x[i])
    wb = bits(inputs.weight_bf16(p.N, p.K, seed=1000 + 16 * (seq.layers - 1) + i, device="cuda"))
    ax, aw = oracle.tensor_scale(xb), oracle.tensor_scale(wb)
    rows = np.unique(np.concatenate([np.random.default_rng(1).choice(seq.tokens, 46, replace=False), [0, 639]]))
    xc, xs = oracle.quantize(np.ascontiguousarray(xb[rows]), ax)
    wc, wsc = oracle.quantize(wb, aw)
    got = bits(seq.y[i])[rows]
    _, err = check_gemm_elementwise(got, oracle.dequantize(xc, xs, ax), oracle.dequantize(wc, wsc, aw), p.K)
    assert err <= 1e-3


def test_graph_replay_with_fused_mlp():
    seq = PrefillSequence(layers=2, tokens=640, device=dev(), mlp=True)
    seq.run()
    torch.cuda.synchronize()
    eager = [None if y is None else bits(y) for y in seq.y]
    seq.capture()
    for y in seq.y:
        if y is not None:
            y.fill_(float("nan"))
    seq.replay()
    torch.cuda.synchronize()
    assert seq.status() == mq.MQ_OK
    for e, y in zip(eager, seq.y):
        if y is not None:
            assert np.array_equal(bits(y), e)
    assert seq.launches() == 2 * (2 * 2 + 5)
    # the last layer's MLP (gate/up weight seed index 2, down index 3) against the oracle
    names = [p.name for p in inputs.QWEN3_8B_PROJECTIONS]
    igu, idn = names.index("gate_up"), names.index("down")
    pgu, pdn = inputs.QWEN3_8B_PROJECTIONS[igu], inputs.QWEN3_8B_PROJECTIONS[idn]
    last = seq.layers - 1
    wgu = bits(inputs.weight_bf16(pgu.N, pgu.K, seed=1000 + 16 * last + igu, device="cuda"))
    wdn = bits(inputs.weight_bf16(pdn.N, pdn.K, seed=1000 + 16 * last + idn, device="cuda"))
    ref = oracle.mlp_w4a4(bits(seq.x[igu]), wgu, wdn)
    got = bits(seq.y[idn])
    assert rel_frobenius(bf16_bits_to_f64(got), bf16_bits_to_f64(ref["y_bf16"])) <= 1e-3
