"""The C-ABI library loads on a machine without a GPU and exports every entry
point that include/*.h declares.  No compute call is made here."""
import glob
import os
import re
import subprocess

import pytest

from selective_state_space_21_b200 import build, scan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"MAMBA_SCAN_API\s+[\w\s\*]*?\b(mamba_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return scan.load_library()


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("mamba_scan_fwd", "mamba_scan_bwd", "mamba_scan_stream_status",
                     "mamba_scan_status_string", "mamba_scan_abi_version"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", scan.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(lib, n)


def test_host_only_entry_points(lib):
    assert lib.mamba_scan_abi_version() == 1
    for code, name in scan.STATUS.items():
        assert lib.mamba_scan_status_string(code).decode() == name
    assert lib.mamba_scan_status_string(99).decode() == "MAMBA_ERR_UNKNOWN"


def test_library_links_no_cuda_driver_or_torch(lib):
    out = subprocess.check_output(["ldd", scan.library_path()], text=True)
    assert "libcuda.so" not in out and "libtorch" not in out and "libc10" not in out


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        scan.mamba_scan_fwd(x, x, None, torch.zeros(2, 4), torch.zeros(1, 4, 8),
                            torch.zeros(1, 4, 8), None, None, torch.zeros_like(x), None)


def test_saved_bytes_queries_check_arguments_on_the_host(lib):
    """The training pairs' size queries refuse a null result pointer and a bad
    rank before touching a device; the projection's pair stores nothing for
    fp32 (the fused kernels take bf16 only), which needs no device either."""
    import ctypes
    n = ctypes.c_uint64(7)
    assert lib.mamba_scan_saved_bytes(2, 64, 128, 16, 1, None, None) == 1
    assert lib.mamba_conv_scan_saved_bytes(2, 64, 128, 16, 4, 1, None, None) == 1
    assert lib.mamba_dtproj_scan_saved_bytes(2, 64, 128, 16, 8, 1, None, None) == 1
    assert lib.mamba_cplx_scan_saved_bytes(2, 64, 128, 8, 1, None) == 1
    assert lib.mamba_dtproj_scan_saved_bytes(2, 64, 128, 16, 0, 1, None, ctypes.byref(n)) == 1
    n.value = 7
    assert lib.mamba_dtproj_scan_saved_bytes(2, 64, 128, 16, 8, 0, None, ctypes.byref(n)) == 0
    assert n.value == 0
