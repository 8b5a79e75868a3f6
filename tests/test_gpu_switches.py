"""The GEMM's tuning switches give the default path's bytes: fewer pipeline
stages (MQ_SWITCH_GEMM_STAGES), another tile raster (MQ_SWITCH_GEMM_GROUP_M)
and launches without programmatic dependent launch (MQ_SWITCH_PDL = 0), set
through mq_set_switch; and the environment sets a switch once, at the first
call into the library (checked in a child process).  Codes, scales and Y are
compared bit for bit with the default path on the same inputs."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_03_b200 import inputs, mq
from tests.gpu_helpers import bits, dev

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
M, K, N = 640, 1024, 1000


def _run():
    """(codes, scales of W; Y of the linear; Y of the MLP) on fixed inputs."""
    x = inputs.activation_bf16(M, K, seed=31, outlier_channels=10, outlier_scale=50.0, device="cuda")
    w = inputs.weight_bf16(N, K, seed=32, device="cuda")
    q = mq.quantize(w)
    lin = mq.LinearW4A4(w)
    y = lin(x)
    mlp = mq.MLPW4A4(inputs.weight_bf16(512, K, seed=33, device="cuda"),
                     inputs.weight_bf16(384, 256, seed=34, device="cuda"))
    y2 = mlp(x)
    torch.cuda.synchronize()
    assert mq.mq_read_status(lin._ws) == mq.MQ_OK
    return (q.codes.cpu().numpy(), q.scales.cpu().numpy(), bits(y), bits(y2))


@pytest.fixture(scope="module")
def default_result():
    return _run()


@pytest.mark.parametrize("values", [{"gemm_stages": 3}, {"gemm_stages": 2}, {"gemm_group_m": 1},
                                    {"gemm_group_m": 5}, {"pdl": 0}],
                         ids=lambda e: ",".join(f"{k}={v}" for k, v in e.items()))
def test_switch_gives_the_default_bytes(values, default_result, switches):
    switches(**values)
    got = _run()
    for a, b in zip(got, default_result):
        assert np.array_equal(a, b)


def test_environment_sets_a_switch_once(default_result, tmp_path):
    """MQ_PDL=0 and MQ_GEMM_STAGES=3 in the environment of a fresh process
    set the switches at the first call; changing the environment afterwards
    changes nothing."""
    out = tmp_path / "y.npz"
    code = ("import os, sys, numpy as np; sys.path.insert(0, %r); "
            "from nvfp4_w4a4_quantized_03_b200 import mq; "
            "assert mq.mq_get_switch('pdl') == 0 and mq.mq_get_switch('gemm_stages') == 3; "
            "os.environ['MQ_PDL'] = '1'; assert mq.mq_get_switch('pdl') == 0; "
            "from tests.test_gpu_switches import _run; r = _run(); "
            "np.savez(%r, *r)") % (ROOT, str(out))
    env = dict(os.environ, MQ_PDL="0", MQ_GEMM_STAGES="3")
    p = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    got = np.load(out)
    for i, b in enumerate(default_result):
        assert np.array_equal(got[f"arr_{i}"], b)
