"""The prefill sequence of linears (nvfp4_w4a4_quantized_03_b200.sequence):
a CUDA-graph replay gives the eager result bit for bit, the shared workspace
reports no device error, and a projection of the last layer matches the
oracle on sampled rows (NVFP4 W4A4 linear, "Mix-Quant：面向智能体LLM的量化预填充
与精确解码", section 方法步骤详情, step (3))."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from nvfp4_w4a4_quantized_03_b200.sequence import PrefillSequence
from tests.gpu_helpers import bf16_bits_to_f64, bits, dev, rel_frobenius

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
    ref = oracle.bf16_rne_array(oracle.gemm_f64(oracle.dequantize(xc, xs, ax), oracle.dequantize(wc, wsc, aw)))
    got = bits(seq.y[i])[rows]
    assert rel_frobenius(bf16_bits_to_f64(got), bf16_bits_to_f64(ref)) <= 1e-3
