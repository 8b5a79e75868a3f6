"""GPU parity of the quantizer (mq_tensor_scale, mq_nvfp4_quantize) against the
CPU oracle: alpha, codes and the whole scale buffer must be bit-exact.

Method: NVFP4 two-level microscaling, "Mix-Quant：面向智能体LLM的量化预填充与精确解码"
(paper.rainbus.top digest), section 方法步骤详情, step (3); r9-hu digest,
section Method, item 1.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import bits, dev, gpu_quantize

pytestmark = pytest.mark.gpu


def _report(name, got, want, x=None):
    bad = np.argwhere(got != want)
    msg = f"{name}: {len(bad)} mismatches"
    for idx in bad[:8]:
        idx = tuple(idx)
        msg += f"\n  at {idx}: gpu {got[idx]:#x} oracle {want[idx]:#x}"
    return msg


def assert_quant_matches(x_cpu, alpha=None):
    rows, K = x_cpu.shape
    a_gpu, codes, scales, _ = gpu_quantize(x_cpu, alpha)
    xb = bits(x_cpu)
    a_ref = oracle.tensor_scale(xb) if alpha is None else float(np.float32(alpha))
    assert a_gpu == a_ref, (a_gpu, a_ref)
    oc, osc = oracle.quantize(xb, a_ref)
    assert np.array_equal(codes, oc), _report("codes", codes, oc)
    stored = oracle.scales_to_stored(osc, K)
    assert np.array_equal(scales, stored), _report("scales", scales, stored)
    return a_gpu, codes, scales


@pytest.mark.parametrize("rows,K", [(1, 64), (3, 128), (128, 1024), (130, 320), (257, 1024),
                                    (1024, 1024), (64, 4096), (33, 12288)])
def test_quantize_activations(rows, K):
    x = inputs.activation_bf16(rows, K, seed=rows + K, outlier_channels=max(1, K // 100), outlier_scale=50.0)
    assert_quant_matches(x)


def test_quantize_weights_cfg_small():
    w = inputs.weight_bf16(1024, 1024, seed=0)
    assert_quant_matches(w)


def test_quantize_student_t():
    x = inputs.student_t_activation_bf16(512, 4096, seed=0)
    a, codes, scales = assert_quant_matches(x)


@pytest.mark.slow
@pytest.mark.parametrize("rows,K", [(8192, 4096), (8192, 12288)])
def test_quantize_full_size(rows, K):
    x = inputs.activation_bf16(rows, K, seed=7, outlier_channels=inputs.outlier_count(K), outlier_scale=50.0)
    assert_quant_matches(x)


def test_tensor_scale_edge_cases():
    ws = mq.workspace(mq.mq_workspace_bytes(), dev())
    alpha = torch.empty(1, dtype=torch.float32, device=dev())
    cases = [torch.zeros(5, 64, dtype=torch.bfloat16),
             torch.tensor([-3.0, 2.0, 1.0], dtype=torch.bfloat16),            # numel not a multiple of 8
             torch.full((1, 13), -0.5, dtype=torch.bfloat16),
             inputs.activation_bf16(777, 64, seed=3)]
    for x in cases:
        mq.mq_tensor_scale(x.to(dev()).contiguous(), alpha, ws)
        torch.cuda.synchronize()
        assert alpha.item() == oracle.tensor_scale(bits(x)), x.shape
    # the workspace counters are back at zero after every call
    assert int(ws[:8].view(torch.int32).abs().sum().item()) == 0


def test_golden_fixture_on_gpu():
    import tests.test_oracle_quant as tq
    a, blocks = tq._load_golden()
    vals = [v for b in blocks for v in b["x"]]
    x = torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16).reshape(1, -1)
    _, codes, scales = assert_quant_matches(x)
    q = oracle.unpack_codes(codes)[0]
    for i, b in enumerate(blocks):
        assert list(q[16 * i:16 * i + 16]) == b["codes"]
        assert scales[oracle.scale_offset(0, i, 128)] == b["scale"]


def test_rounding_midpoints_sweep():
    """Blocks whose scale quotient t and element quotients v sit on, and within
    a few ulps of, every E4M3 and E2M1 midpoint (alpha is perturbed by a few
    binary32 ulps around 2^-4 so that fl32 arithmetic lands on each side)."""
    mids_e4m3 = []
    for c in range(0x7E):
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        mids_e4m3.append(0.5 * (lo + hi))
    rows = []
    for m in mids_e4m3:
        amax_b = m * 0.375          # t = amax_b / (6 * 2^-4) = m; exact in bf16 for these m
        blk = [amax_b] + [amax_b * f for f in (0.0417, 0.125, 0.208, 0.29, 0.375, 0.458, 0.583,
                                               0.708, 0.8333, -0.0417, -0.29, -0.583, -0.8333, -1.0, 0.5)]
        rows.append(blk)
    rows += [[0.375 * 16 * v / 6.0 for v in (6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75,
                                             -1.25, -1.75, -2.5, -3.5, -5.0, 0.125)]] * 2
    x = torch.tensor(rows, dtype=torch.float64).to(torch.bfloat16).reshape(-1, 64)
    for k in range(-4, 5):
        alpha = float(np.float32(2.0 ** -4) * np.float32(1 + k * 2.0 ** -23))
        assert_quant_matches(x, alpha=alpha)


@pytest.mark.slow
def test_repeated_runs_match_the_oracle():
    """The quantizers stream X through a ring of shared-memory slots that TMA
    refills while other warps still quantize: repeated runs on an activation
    that gives each block ~20 boxes (8192 x 12288) must all match the
    oracle, every L2 state included (a flush before every other run), and the
    linear's one-pass quantizer must give the same Y every time."""
    rows, K = 8192, 12288
    x_cpu = inputs.activation_bf16(rows, K, seed=77, outlier_channels=inputs.outlier_count(K), outlier_scale=50.0)
    a0, codes0, scales0 = assert_quant_matches(x_cpu)
    x = x_cpu.to(dev())
    q = mq.QuantizedTensor(rows, K, dev())
    q.alpha.fill_(a0)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev())
    for r in range(12):
        if r % 2:
            flush.sum()
        q.codes.zero_()
        mq.mq_nvfp4_quantize(x, q.alpha, q.codes, q.scales)
        torch.cuda.synchronize()
        assert np.array_equal(q.codes.cpu().numpy().reshape(rows, K // 2), codes0), r
        assert np.array_equal(q.scales.cpu().numpy(), scales0), r
    lin = mq.LinearW4A4(inputs.weight_bf16(1024, K, seed=78, device=dev()))
    y0 = lin(x).clone()
    for r in range(12):
        if r % 2:
            flush.sum()
        assert torch.equal(lin(x).view(torch.int16), y0.view(torch.int16)), r
    assert mq.mq_read_status(lin._ws) == mq.MQ_OK


def test_codes_buffer_16_byte_aligned():
    """A codes buffer that is 16- but not 32-byte aligned (the ABI asks for
    16) takes the two 128-bit stores per quad instead of one 256-bit store:
    the same bytes."""
    rows, K = 640, 1024
    x_cpu = inputs.activation_bf16(rows, K, seed=91, outlier_channels=10, outlier_scale=50.0)
    a0, codes0, scales0 = assert_quant_matches(x_cpu)
    x = x_cpu.to(dev())
    q = mq.QuantizedTensor(rows, K, dev())
    q.alpha.fill_(a0)
    n = mq.mq_nvfp4_codes_bytes(rows, K)
    buf = torch.zeros(n + 64, dtype=torch.uint8, device=dev())
    off = 16 if buf.data_ptr() % 32 == 0 else 32      # 16 mod 32 either way
    codes = buf[off:off + n]
    assert codes.data_ptr() % 32 == 16
    mq.mq_nvfp4_quantize(x, q.alpha, codes, q.scales)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy().reshape(rows, K // 2), codes0)
    assert np.array_equal(q.scales.cpu().numpy(), scales0)
