"""Token and column sharding of the W4A4 linear on one GPU.

Token sharding: max|x| per shard
(mq_tensor_amax), the maximum over shards (the step an NCCL all-reduce takes
across GPUs), alpha from it (mq_alpha_from_amax), then each shard quantized
and multiplied: the rows equal those of mq_linear_w4a4 on the whole
activation bit for bit, and alpha equals the oracle's tensor-level scale of
the whole activation ("张量级尺度", section NVFP4 微缩放量化 of the
paper.rainbus.top digest).

Column sharding: each shard of the weight's rows quantized under the whole
weight's alpha (max|w| per shard, the maximum over shards), then the linear
on the full activation: the columns equal those of the unsharded linear bit
for bit (prefill-shaped M, whose GEMM sums every output over K in one fixed
order whatever N is)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from nvfp4_w4a4_quantized_03_b200.sharded import ColumnShardedLinearW4A4, ShardedLinearW4A4
from tests.gpu_helpers import bits, dev

pytestmark = pytest.mark.gpu


def _amax_def(x_cpu):
    """max |x| by its definition, on the bf16 bit patterns."""
    b = bits(x_cpu).astype(np.uint32) & 0x7FFF
    return float((np.max(b) << 16).astype(np.uint32).view(np.float32)) if b.size else 0.0


@pytest.mark.parametrize("shape", [(1, 8), (3, 5), (7, 1000), (128, 4096), (1000, 12288)])
def test_tensor_amax_is_max_abs(shape):
    x = inputs.activation_bf16(*shape, seed=sum(shape), outlier_channels=1, outlier_scale=50.0)
    amax = torch.zeros(1, dtype=torch.float32, device=dev())
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    mq.mq_tensor_amax(x.to(dev()), amax, ws)
    assert float(amax.item()) == _amax_def(x)
    mq.mq_tensor_amax(torch.zeros(shape, dtype=torch.bfloat16, device=dev()), amax, ws)
    assert float(amax.item()) == 0.0


@pytest.mark.parametrize("a", [0.0, 1.0, 2688.0, 3.0e-5, 168.0, 65280.0, 1.0e-38])
def test_alpha_from_amax(a):
    amax = torch.tensor([a], dtype=torch.float32, device=dev())
    alpha = torch.zeros(1, dtype=torch.float32, device=dev())
    mq.mq_alpha_from_amax(amax, alpha)
    want = 1.0 if a == 0.0 else float(np.float32(a) / np.float32(2688.0))
    assert float(alpha.item()) == want


def test_shards_equal_the_whole_linear():
    M, K, N = 1000, 4096, 2048
    x = inputs.activation_bf16(M, K, seed=11, outlier_channels=41, outlier_scale=50.0).to(dev())
    w = inputs.weight_bf16(N, K, seed=12).to(dev())
    lin = mq.LinearW4A4(w)
    y_whole = lin(x)
    cuts = [(0, 300), (300, 301), (301, 1000)]
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    amaxes = []
    for a, b in cuts:
        t = torch.zeros(1, dtype=torch.float32, device=dev())
        mq.mq_tensor_amax(x[a:b], t, ws)
        amaxes.append(t)
    amax = torch.stack(amaxes).max().reshape(1)    # the all-reduce's result
    ys = []
    for a, b in cuts:
        q = mq.QuantizedTensor(b - a, K, dev())
        mq.mq_alpha_from_amax(amax, q.alpha)
        mq.mq_nvfp4_quantize(x[a:b], q.alpha, q.codes, q.scales)
        y = torch.empty(b - a, N, dtype=torch.bfloat16, device=dev())
        mq.mq_nvfp4_gemm(q.codes, q.scales, q.alpha, lin.w.codes, lin.w.scales, lin.w.alpha, b - a, N, K, y, ws)
        ys.append(y)
        assert float(q.alpha.item()) == oracle.tensor_scale(bits(x))
    torch.cuda.synchronize()
    assert np.array_equal(bits(torch.cat(ys)), bits(y_whole))


def test_sharded_linear_single_rank_is_the_linear():
    M, K, N = 256, 1024, 768
    x = inputs.activation_bf16(M, K, seed=3, outlier_channels=10, outlier_scale=50.0).to(dev())
    w = inputs.weight_bf16(N, K, seed=4).to(dev())
    y1 = ShardedLinearW4A4(w)(x)
    y2 = mq.LinearW4A4(w)(x)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y1), bits(y2))


def test_column_shards_equal_the_whole_linear():
    M, K, N = 1000, 4096, 2048
    x = inputs.activation_bf16(M, K, seed=21, outlier_channels=41, outlier_scale=50.0).to(dev())
    w = inputs.weight_bf16(N, K, seed=22).to(dev())
    lin = mq.LinearW4A4(w)
    y_whole = lin(x)
    cuts = [(0, 768), (768, 1468), (1468, 2048)]          # one cut off the 128-row tiles
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    amaxes = []
    for a, b in cuts:
        t = torch.zeros(1, dtype=torch.float32, device=dev())
        mq.mq_tensor_amax(w[a:b].contiguous(), t, ws)
        amaxes.append(t)
    amax = torch.stack(amaxes).max().reshape(1)    # the all-reduce's result
    wc_whole = lin.w.codes.cpu().numpy().reshape(N, K // 2)
    ws_whole = oracle.scales_from_stored(lin.w.scales.cpu().numpy(), N, K)
    for a, b in cuts:
        q = mq.QuantizedTensor(b - a, K, dev())
        mq.mq_alpha_from_amax(amax, q.alpha)
        mq.mq_nvfp4_quantize(w[a:b].contiguous(), q.alpha, q.codes, q.scales)
        assert float(q.alpha.item()) == float(lin.w.alpha.item())
        assert np.array_equal(q.codes.cpu().numpy().reshape(b - a, K // 2), wc_whole[a:b])
        assert np.array_equal(oracle.scales_from_stored(q.scales.cpu().numpy(), b - a, K), ws_whole[a:b])
        y = torch.empty(M, b - a, dtype=torch.bfloat16, device=dev())
        lws = mq.workspace(mq.mq_linear_w4a4_workspace_bytes(M, K), dev())
        mq.mq_linear_w4a4(x, q.codes, q.scales, q.alpha, b - a, y, lws)
        torch.cuda.synchronize()
        assert np.array_equal(bits(y), bits(y_whole[:, a:b]))


def test_column_sharded_single_rank_is_the_linear():
    M, K, N = 300, 1024, 640
    x = inputs.activation_bf16(M, K, seed=23, outlier_channels=10, outlier_scale=50.0).to(dev())
    w = inputs.weight_bf16(N, K, seed=24).to(dev())
    y1 = ColumnShardedLinearW4A4(w)(x)
    y2 = mq.LinearW4A4(w)(x)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y1), bits(y2))
