"""The bounds-check build (libmq_debug.so, MQ_DEBUG=1), the stand-in for a
memory checker: the workloads below run in a child process on the debug
build, which checks every index-computed global access and every TMA
coordinate before it is made.  No check may fail, and every output must
equal the release library's bit for bit (the checks only guard accesses).

Workloads: quantizer on ragged shapes; the GEMM's one-CTA, pair and decode
forms on ragged shapes; the linear's three quantization paths; the MLP."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _workloads():
    """Outputs of every workload as a list of uint8/uint16 arrays; runs on
    whichever library the binding loaded (MQ_DEBUG selects it)."""
    import torch

    from nvfp4_w4a4_quantized_03_b200 import inputs, mq
    out = []
    b16 = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    for rows, K in [(1, 64), (130, 320), (257, 1024), (1000, 4096)]:
        q = mq.quantize(inputs.activation_bf16(rows, K, seed=rows + K, outlier_channels=3, device="cuda"))
        out += [q.codes.cpu().numpy(), q.scales.cpu().numpy()]
    for M, N, K, form in [(3, 17, 128, None), (64, 4096, 4096, None), (130, 300, 320, "1"), (257, 513, 1024, "2"),
                          (700, 1024, 4096, None)]:
        qx = mq.quantize(inputs.activation_bf16(M, K, seed=M, outlier_channels=3, device="cuda"))
        qw = mq.quantize(inputs.weight_bf16(N, K, seed=N, device="cuda"))
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        with mq.switch(gemm_form=int(form or 0)):
            mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, qw.codes, qw.scales, qw.alpha, M, N, K, y)
        out.append(b16(y))
    M, K, N = 300, 1024, 768
    x = inputs.activation_bf16(M, K, seed=9, outlier_channels=10, device="cuda")
    lin = mq.LinearW4A4(inputs.weight_bf16(N, K, seed=10, device="cuda"))
    for path in ("onepass", "split", "ingemm"):
        with mq.switch(linear_path=path):
            out.append(b16(lin(x)))
    mlp = mq.MLPW4A4(inputs.weight_bf16(512, K, seed=11, device="cuda"), inputs.weight_bf16(384, 256, seed=12,
                                                                                         device="cuda"))
    out.append(b16(mlp(x)))
    torch.cuda.synchronize()
    return out


def test_debug_build_checks_pass_and_match_the_release_build(tmp_path):
    from nvfp4_w4a4_quantized_03_b200 import mq
    assert not mq.mq_is_debug_build()
    release = _workloads()
    out = tmp_path / "dbg.npz"
    code = ("import sys, numpy as np; sys.path.insert(0, %r); "
            "from nvfp4_w4a4_quantized_03_b200 import mq; assert mq.mq_is_debug_build(); "
            "from tests.test_gpu_debug_build import _workloads; r = _workloads(); "
            "np.savez(%r, hits=np.array([mq.mq_debug_bounds_hits()]), *r)") % (ROOT, str(out))
    env = dict(os.environ, MQ_DEBUG="1")
    p = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert p.returncode == 0, p.stderr[-3000:]
    got = np.load(out)
    assert int(got["hits"][0]) == 0
    for i, r in enumerate(release):
        assert np.array_equal(got[f"arr_{i}"], r), i
