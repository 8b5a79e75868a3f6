import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU or GPU case")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


_BRUTE_SRC = os.path.join(ROOT, "tests", "pins", "brute_round.c")


@pytest.fixture(scope="session")
def brute(tmp_path_factory):
    """The test-side brute-force rounding checker (tests/pins/brute_round.c)."""
    out = str(tmp_path_factory.mktemp("brute") / "libbrute.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                           "-ffp-contract=off", "-o", out, _BRUTE_SRC, "-lm"])
    lib = ctypes.CDLL(out)
    lib.brute_e2m1.argtypes = [ctypes.c_float]
    lib.brute_e2m1.restype = ctypes.c_uint8
    lib.brute_e4m3.argtypes = [ctypes.c_float]
    lib.brute_e4m3.restype = ctypes.c_uint8
    lib.brute_count_mismatch.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64,
                                         ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint32)]
    lib.brute_count_mismatch.restype = ctypes.c_uint64
    return lib


@pytest.fixture
def switches():
    """Sets libmq's process-wide switches (mq.mq_set_switch) for one test and
    restores every switch afterwards: `switches(gemm_form=2)`."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    saved = {name: mq.mq_get_switch(name) for name in mq.SWITCHES}

    def set_(**values):
        for name, v in values.items():
            mq.mq_set_switch(name, v)

    yield set_
    for name, v in saved.items():
        mq.mq_set_switch(name, v)
