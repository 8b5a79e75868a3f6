"""The C-ABI library builds, loads and exports every entry point that
include/mq.h declares; host-side argument checks answer without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(mq_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def libmq():
    from nvfp4_w4a4_quantized_03_b200 import build, mq
    build.build()
    return mq.lib()


def test_header_declares_the_path():
    names = set(_declared_functions())
    for required in ("mq_tensor_scale", "mq_nvfp4_quantize", "mq_nvfp4_gemm", "mq_linear_w4a4"):
        assert required in names


def test_every_declared_symbol_is_exported(libmq):
    from nvfp4_w4a4_quantized_03_b200 import mq
    out = subprocess.run(["nm", "-D", "--defined-only", mq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(mq_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    for n in _declared_functions():
        getattr(libmq, n)


def test_sizes(libmq):
    from nvfp4_w4a4_quantized_03_b200 import mq
    assert mq.mq_nvfp4_codes_bytes(8192, 4096) == 8192 * 2048
    assert mq.mq_nvfp4_scales_bytes(8192, 4096) == 8192 * 256
    assert mq.mq_nvfp4_scales_bytes(1, 64) == 128 * 4
    assert mq.mq_nvfp4_scales_bytes(130, 320) == 256 * 20
    assert mq.mq_workspace_bytes() == 256
    # header | readiness flags (1 row tile x 4 K stages, padded to 256 B) | codes | scales
    assert mq.mq_linear_w4a4_workspace_bytes(128, 1024) == 256 + 256 + 65536 + 8192
    # the linear's workspace | H bf16 | codes of H | scales of H
    assert mq.mq_mlp_w4a4_workspace_bytes(128, 1024, 256) == 74240 + 65536 + 16384 + 2048


def test_host_validation_without_gpu(libmq):
    """Bad arguments are refused before any device call."""
    vp = ctypes.c_void_p
    p16 = vp(4096)          # an aligned dummy address; never dereferenced
    assert libmq.mq_nvfp4_quantize(p16, 128, 100, p16, p16, p16, None) == -2      # K % 64
    assert libmq.mq_nvfp4_quantize(p16, 0, 128, p16, p16, p16, None) == -2        # rows
    assert libmq.mq_nvfp4_quantize(None, 1, 64, p16, p16, p16, None) == -1        # null
    assert libmq.mq_nvfp4_quantize(vp(4097), 1, 64, p16, p16, p16, None) == -3    # misaligned
    assert libmq.mq_tensor_scale(p16, 64, p16, p16, 16, None) == -5                # workspace too small
    assert libmq.mq_tensor_amax(p16, 64, p16, p16, 16, None) == -5                 # workspace too small
    assert libmq.mq_tensor_amax(None, 64, p16, p16, 256, None) == -1               # null
    assert libmq.mq_tensor_amax(vp(4097), 64, p16, p16, 256, None) == -3           # misaligned
    assert libmq.mq_alpha_from_amax(None, p16, None) == -1                         # null
    assert libmq.mq_alpha_from_amax(vp(4097), p16, None) == -3                     # misaligned
    assert libmq.mq_linear_w4a4(p16, 128, 1024, p16, p16, p16, 256, p16, p16, 1024, None) == -5
    assert libmq.mq_nvfp4_gemm(p16, p16, p16, p16, p16, p16, 1, 1, 96, p16, None, 0, None) == -2
    # gate/up GEMM with SwiGLU: inter a multiple of 128, h_amax required and 4-byte aligned
    assert libmq.mq_nvfp4_gemm_swiglu(p16, p16, p16, p16, p16, p16, 256, 100, 1024, p16, p16, None, 0, None) == -2
    assert libmq.mq_nvfp4_gemm_swiglu(p16, p16, p16, p16, p16, p16, 256, 128, 1024, p16, None, None, 0, None) == -1
    assert libmq.mq_nvfp4_gemm_swiglu(p16, p16, p16, p16, p16, p16, 256, 128, 1024, p16, vp(4098), None, 0,
                                      None) == -3
    assert libmq.mq_nvfp4_gemm_swiglu(p16, p16, p16, p16, p16, p16, 256, 128, 96, p16, p16, None, 0, None) == -2
    # the MLP: workspace size, inter a multiple of 128
    assert libmq.mq_mlp_w4a4(p16, 128, 1024, p16, p16, p16, 256, p16, p16, p16, 64, p16, p16, 1024, None) == -5
    assert libmq.mq_mlp_w4a4(p16, 128, 1024, p16, p16, p16, 64, p16, p16, p16, 64, p16, p16, 1 << 30, None) == -2
    assert libmq.mq_mlp_w4a4(p16, 128, 1024, None, p16, p16, 256, p16, p16, p16, 64, p16, p16, 1 << 30, None) == -1
    assert libmq.mq_status_string(-7) == b"MQ_ERR_TIMEOUT"


def test_noalloc_constant_and_host_checks(libmq):
    """The binding's scratch size is the header's, and the allocation-free
    linear refuses bad shapes before it touches the device: the shape limits of
    mq_linear_w4a4 come first, then the scratch size."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    text = open(os.path.join(HEADER_DIR, "mq.h")).read()
    m = re.search(r"#define\s+MQ_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "MQ_NOALLOC_SCRATCH_BYTES not found in mq.h"
    assert mq.MQ_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
    f = libmq.mq_linear_w4a4_noalloc
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp]
    f.restype = ctypes.c_int
    p16 = vp(4096)
    assert f(p16, 128, 100, p16, p16, p16, 256, p16, None) == -2                 # K % 64
    assert f(p16, 128, 1024, p16, p16, p16, (1 << 31) + 1, p16, None) == -2      # N beyond the row limit
    assert f(p16, 1 << 40, 1 << 20, p16, p16, p16, 256, p16, None) == -2         # M * K beyond the 32-bit block index
    assert f(None, 128, 1024, p16, p16, p16, 256, p16, None) == -1               # null
    assert f(vp(4097), 128, 1024, p16, p16, p16, 256, p16, None) == -3           # misaligned
    assert f(p16, 131072, 4096, p16, p16, p16, 256, p16, None) == -5             # beyond the scratch


def test_debug_build_exports_the_same_symbols(libmq):
    """libmq_debug.so (the MQ_DEBUG bounds-check build) exports every
    declared entry point and reports itself as the debug build."""
    from nvfp4_w4a4_quantized_03_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.DEBUG_LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(mq_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    dbg = ctypes.CDLL(build.DEBUG_LIB)
    assert dbg.mq_is_debug_build() == 1
    assert libmq.mq_is_debug_build() == 0


def test_switches_without_gpu(libmq):
    """The switch table answers on the host: defaults (or the environment's
    values), range checks that keep the old value, and the numbering of
    mq.h's MQ_SWITCH_* enumerators."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    text = open(os.path.join(HEADER_DIR, "mq.h")).read()
    enum = dict((k, int(v)) for k, v in re.findall(r"MQ_SWITCH_([A-Z_]+)\s*=\s*(\d+)", text))
    assert enum.pop("COUNT") == len(mq.SWITCHES)
    assert {k.lower(): v for k, v in enum.items()} == mq.SWITCHES
    saved = {n: mq.mq_get_switch(n) for n in mq.SWITCHES}
    try:
        for name, good, bad in [("linear_path", 2, 3), ("gemm_form", 1, 3), ("gemm_decode", 0, 2),
                                ("decode_split", 8, 3), ("gemm_stages", 2, 1), ("gemm_group_m", 7, -1),
                                ("pdl", 0, 2)]:
            mq.mq_set_switch(name, good)
            assert mq.mq_get_switch(name) == good
            assert libmq.mq_set_switch(mq.SWITCHES[name], bad) == -1       # MQ_ERR_INVALID_ARG
            assert mq.mq_get_switch(name) == good
        assert libmq.mq_get_switch(len(mq.SWITCHES)) == -1
        assert libmq.mq_set_switch(-1, 0) == -1
        with mq.switch(linear_path="split", gemm_form=2):
            assert mq.mq_get_switch("linear_path") == 1 and mq.mq_get_switch("gemm_form") == 2
        assert mq.mq_get_switch("linear_path") == 2 and mq.mq_get_switch("gemm_form") == 1
    finally:
        for n, v in saved.items():
            mq.mq_set_switch(n, v)


def test_switches_read_from_the_environment_once(libmq):
    """A fresh process takes each switch from its environment variable at the
    first call (names or numbers for the linear path; invalid values keep the
    default) and ignores later changes of the environment."""
    import sys
    code = ("import os, sys; sys.path.insert(0, %r); "
            "from nvfp4_w4a4_quantized_03_b200 import mq; "
            "print([mq.mq_get_switch(n) for n in ('linear_path', 'decode_split', 'gemm_stages', 'pdl', 'gemm_form')]); "
            "os.environ['MQ_PDL'] = '1'; print(mq.mq_get_switch('pdl'))") % ROOT
    env = dict(os.environ, MQ_LINEAR_PATH="ingemm", MQ_DECODE_SPLIT="3", MQ_GEMM_STAGES="1", MQ_PDL="0",
               MQ_GEMM_FORM="2")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.split("\n")
    assert lines[0] == "[2, 0, 0, 0, 2]", out.stdout
    assert lines[1] == "0", out.stdout
    env["MQ_LINEAR_PATH"] = "1"
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert out.stdout.split("\n")[0] == "[1, 0, 0, 0, 2]", out.stdout
