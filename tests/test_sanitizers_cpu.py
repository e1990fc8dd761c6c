"""AddressSanitizer and UndefinedBehaviorSanitizer over the host-side code
that runs without a GPU: the fp64 oracle (every entry point, including
empty and one-step problems) and the C ABI's argument checks (every entry
point with invalid arguments).  Each runs in a child process with the ASan
runtime preloaded; any report fails the test.  No GPU is involved: on a
machine without one the ABI's calls stop at their argument checks or at the
first CUDA call (MAMBA_ERR_CUDA)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ASAN_RT = "/usr/lib/x86_64-linux-gnu/libasan.so.8"

pytestmark = pytest.mark.skipif(not os.path.exists(ASAN_RT), reason="no ASan runtime")


def _run(script: str, *args) -> subprocess.CompletedProcess:
    env = dict(os.environ)
    env["LD_PRELOAD"] = ASAN_RT
    env["ASAN_OPTIONS"] = "detect_leaks=0:halt_on_error=1:abort_on_error=0"
    env["UBSAN_OPTIONS"] = "halt_on_error=1:print_stacktrace=1"
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    env["CUDA_VISIBLE_DEVICES"] = ""  # host paths only, even on a machine with a GPU
    return subprocess.run([sys.executable, "-c", script, *args], env=env, capture_output=True,
                          text=True, timeout=600)


def _check(r: subprocess.CompletedProcess):
    out = r.stdout + r.stderr
    assert "AddressSanitizer" not in out and "runtime error" not in out, out[-4000:]
    assert r.returncode == 0, out[-4000:]


ORACLE_SCRIPT = r"""
import sys
import numpy as np
import torch
import oracle
from selective_state_space_21_b200.inputs import (make_inputs, make_conv_params,
                                                  make_dtproj_params, make_cplx_inputs)
lib = oracle.load_library(sys.argv[1])
for (b, d, L, N) in [(1, 3, 17, 4), (2, 2, 1, 1), (1, 1, 0, 3), (0, 2, 5, 2), (2, 5, 33, 16)]:
    x = make_inputs(b, d, L, N, torch.float32, seed=3, with_dy=True)
    y, last = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                x["D"], x["z"], lib=lib)
    g = oracle.s6_backward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"], x["delta_bias"],
                           x["D"], x["z"], lib=lib)
    y2, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], None, None, None,
                              nthreads=3, lib=lib)
    if b * d * L:
        cp = make_conv_params(d, 4, seed=1)
        oracle.s6_conv_forward(x["u"], cp["conv_w"], cp["conv_b"], x["delta"], x["A"], x["B"],
                               x["C"], x["delta_bias"], x["D"], x["z"], lib=lib)
        oracle.s6_conv_backward(x["u"], cp["conv_w"], cp["conv_b"], x["delta"], x["A"], x["B"],
                                x["C"], x["dy"], x["delta_bias"], x["D"], x["z"], lib=lib)
        pp = make_dtproj_params(b, d, L, 3, torch.float32, seed=2)
        oracle.s6_dtproj_forward(x["u"], pp["dt_low"], pp["W_dt"], x["A"], x["B"], x["C"],
                                 x["delta_bias"], x["D"], x["z"], lib=lib)
        oracle.s6_dtproj_backward(x["u"], pp["dt_low"], pp["W_dt"], x["A"], x["B"], x["C"],
                                  x["dy"], x["delta_bias"], x["D"], x["z"], lib=lib)
        cx = make_cplx_inputs(b, d, L, N, torch.float32, seed=4, with_dy=True)
        oracle.s6_cplx_forward(cx["u"], cx["delta"], cx["A"], cx["B"], cx["C"],
                               cx["delta_bias"], cx["D"], cx["z"], lib=lib)
        oracle.s6_cplx_backward(cx["u"], cx["delta"], cx["A"], cx["B"], cx["C"], cx["dy"],
                                cx["delta_bias"], cx["D"], cx["z"], lib=lib)
print("oracle ok")
"""


def test_oracle_under_asan_and_ubsan(tmp_path):
    """The oracle compiled with -fsanitize=address,undefined runs every entry
    point, empty and degenerate shapes included, without a report."""
    import oracle
    so = str(tmp_path / "libs6oracle_asan.so")
    subprocess.check_call(["gcc", "-O1", "-g", "-fno-omit-frame-pointer", "-fsanitize=address",
                           "-fsanitize=undefined", "-fno-sanitize-recover=undefined",
                           "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
                           "-pthread", oracle._SRC, "-o", so, "-lm"])
    r = _run(ORACLE_SCRIPT, so)
    _check(r)
    assert "oracle ok" in r.stdout


ABI_SCRIPT = r"""
import ctypes, sys
lib = ctypes.CDLL(sys.argv[1])
vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
buf = ctypes.create_string_buffer(1 << 16)
h = ctypes.cast(buf, vp)   # host memory: never accepted as a tensor
def call(name, *args):
    f = getattr(lib, name)
    f.restype = ctypes.c_int
    return f(*args)
codes = []
# forward / backward: bad N, dtype, sizes, options, host pointers
opts = (ctypes.c_int32 * 8)(9, 0, 0, 0, 0, 0, 0, 0)  # path out of range
fwd = [h, h, None, h, h, h, None, None, h, None]
for (b, d, L, N, dt) in [(1, 2, 8, 17, 0), (1, 2, 8, 4, 7), (-1, 2, 8, 4, 0), (1, 2, 8, 4, 0),
                         (0, 0, 0, 4, 1), (70000, 2, 8, 4, 0), (1, 2, 8, 0, 0)]:
    codes.append(call("mamba_scan_fwd", *fwd, i64(b), i64(d), i64(L), i64(N), i32(dt), None))
    codes.append(call("mamba_scan_fwd_ex", *fwd, i64(b), i64(d), i64(L), i64(N), i32(dt),
                      ctypes.byref(opts), None))
    codes.append(call("mamba_scan_fwd_noalloc", *fwd, i64(b), i64(d), i64(L), i64(N), i32(dt), None))
    bwd = [h, h, None, h, h, h, None, None, h, h, h, h, h, h, None, None, None]
    codes.append(call("mamba_scan_bwd", *bwd, i64(b), i64(d), i64(L), i64(N), i32(dt), None))
    codes.append(call("mamba_cplx_scan_fwd", *fwd, i64(b), i64(d), i64(L), i64(N), i32(dt), None))
    codes.append(call("mamba_cplx_scan_bwd", *bwd, i64(b), i64(d), i64(L), i64(N), i32(dt), None))
    codes.append(call("mamba_scan_step", h, h, h, None, h, h, h, None, None, h, i64(b), i64(d),
                      i64(N), i32(dt), None))
    for W in (0, 3, 5):
        codes.append(call("mamba_conv_scan_fwd", h, h, None, i64(W), h, None, h, h, h, None, None,
                          h, None, i64(b), i64(d), i64(L), i64(N), i32(dt), None, None))
        codes.append(call("mamba_conv_scan_step", h, h, h, h, None, i64(W), h, None, h, h, h,
                          None, None, h, i64(b), i64(d), i64(N), i32(dt), None))
    for R in (0, 3, 1 << 21):
        codes.append(call("mamba_dtproj_scan_fwd", h, h, h, i64(R), None, h, h, h, None, None, h,
                          None, i64(b), i64(d), i64(L), i64(N), i32(dt), None, None))
plan = vp()
codes.append(call("mamba_scan_step_plan_create", ctypes.byref(plan), h, h, h, None, None, i64(0),
                  h, None, h, h, h, None, None, h, i64(1), i64(2), i64(4), i32(0)))
codes.append(call("mamba_scan_step_plan_create", None, h, None, h, None, None, i64(0),
                  h, None, h, h, h, None, None, h, i64(1), i64(2), i64(4), i32(0)))
codes.append(call("mamba_scan_step_plan_run", None, None))
lib.mamba_scan_step_plan_destroy(None)
codes.append(call("mamba_scan_pool_set_reserve", ctypes.c_uint64(0)))
codes.append(call("mamba_scan_pool_trim", ctypes.c_uint64(0)))
r = ctypes.c_uint64()
codes.append(call("mamba_scan_pool_reserved", ctypes.byref(r)))
codes.append(call("mamba_scan_pool_reserved", None))
lib.mamba_scan_test_fail_alloc(i32(2))
lib.mamba_scan_test_fail_alloc(i32(-1))
codes.append(call("mamba_scan_stream_status", None))
lib.mamba_scan_status_string.restype = ctypes.c_char_p
names = [lib.mamba_scan_status_string(i32(c)) for c in range(-1, 8)]
assert all(n is not None for n in names)
assert all(c in (0, 1, 2, 3) for c in codes), codes
assert 0 not in codes[:3], codes
print("abi ok", len(codes))
"""


@pytest.fixture(scope="module")
def asan_library(tmp_path_factory):
    """libmambascan with ASan and UBSan in its host code (device code as PTX
    only: nothing is launched here)."""
    out = str(tmp_path_factory.mktemp("asan") / "libmambascan_asan.so")
    from selective_state_space_21_b200 import build
    cmd = [build.NVCC, "-gencode", "arch=compute_100a,code=compute_100a", "-O1", "-g",
           "-std=c++17", "--expt-relaxed-constexpr", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fsanitize=address", "-Xcompiler", "-fsanitize=undefined",
           "-Xcompiler", "-fno-sanitize-recover=undefined", "-Xcompiler",
           "-fno-omit-frame-pointer", "-cudart", "static", "-I", os.path.join(ROOT, "include"),
           *build.sources(), "-o", out]
    subprocess.check_call(cmd, timeout=1200)
    return out


def test_abi_argument_checks_under_asan_and_ubsan(asan_library):
    """Every entry point of the C ABI, called with invalid arguments (sizes out
    of range, N outside 1..16, a bad dtype, options out of range,
    convolution widths and ranks out of range, host pointers, null
    handles), returns an error code without an ASan or UBSan report."""
    r = _run(ABI_SCRIPT, asan_library)
    _check(r)
    assert "abi ok" in r.stdout
