"""The small GPU parity cases again, against the bounds-checking build of the
library (libmambascan_debug.so, compiled with MAMBA_DEBUG_BOUNDS): there every
kernel checks the indices it computes into its workspace and its outputs
against the buffers' sizes, skips an access outside them and records it in
the sticky status, which the parity helpers read after every call
(MAMBA_ERR_OUT_OF_BOUNDS fails the case).  compute-sanitizer being closed on
this pool, this build is how the index arithmetic is checked on the GPU.  The
cases run in a child pytest process that loads the debug library through
MAMBA_SCAN_LIBRARY."""
import os
import subprocess
import sys

import pytest
import torch

from selective_state_space_21_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# every small-shape case: staged grids, chunkings and carries, random shapes,
# the convolution prologue, the projection, complex A, decoding, the limits
SELECT = "not full_workload and not full_size and not wait_times_out and not many_channels"
FILES = ["tests/test_parity_gpu.py", "tests/test_parity_conv_gpu.py",
         "tests/test_parity_dtproj_gpu.py", "tests/test_parity_decode_gpu.py",
         "tests/test_parity_limits_gpu.py", "tests/test_parity_cplx_gpu.py"]


def test_parity_cases_pass_under_bounds_checks():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = build.build_debug()
    env = dict(os.environ, MAMBA_SCAN_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-k", SELECT,
                        "-p", "no:cacheprovider", *FILES], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=3600)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
