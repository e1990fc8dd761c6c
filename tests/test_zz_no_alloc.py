"""The allocation-free forward, mamba_scan_fwd_noalloc, against the regular
forward, mamba_scan_fwd, through the C ABI.

That entry point exists for callers that cannot let a library allocate device
memory (their own allocator owns it, or allocation calls are not allowed where
they run); it keeps its scratch in a fixed per-device array instead.  Each case
runs it twice in a row, so the second call sees the array as the first left it.
This file is collected last on purpose, and passes both alone in a fresh
process (the first call on the device sets the array up) and after the other
tests.
"""
import pytest
import torch

import gpu_cases as gc
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import make_inputs, workload_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()


def _regular(x):
    y = torch.empty_like(x["u"])
    last = torch.empty(x["u"].shape[0], x["u"].shape[1], x["A"].shape[1], device="cuda")
    scan.mamba_scan_fwd(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"],
                        x["z"], y, last)
    assert scan.mamba_scan_stream_status() == 0
    return y, last


def _noalloc_twice(x):
    """Two calls in a row, each with the library's allocation-failure hook
    armed (any workspace allocation the call made would fail it with
    MAMBA_ERR_OUT_OF_MEMORY) and with its workspace pool emptied first (the
    call must leave it empty)."""
    out = []
    for _ in range(2):
        y = torch.full_like(x["u"], float("nan"))
        last = torch.full((x["u"].shape[0], x["u"].shape[1], x["A"].shape[1]), float("nan"),
                          device="cuda")
        torch.cuda.synchronize()
        scan.pool_trim(0)
        reserved0 = scan.pool_reserved()
        scan.test_fail_alloc(0)
        try:
            scan.mamba_scan_fwd_noalloc(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"],
                                        x["C"], x["D"], x["z"], y, last)
        finally:
            scan.test_fail_alloc(-1)
        assert scan.mamba_scan_stream_status() == 0
        assert scan.pool_reserved() == reserved0 == 0
        out.append((y, last))
    return out


CASES = [  # (batch, dim, L, N, dtype): chunked hand-off, several group counts, N rounding,
    (8, 5120, 2048, 16, torch.bfloat16),  # the full bf16 2K-length workload
    (1, 1536, 65536, 16, torch.bfloat16),  # few groups, long: chunks from zero, scan, correction
    (2, 300, 1024, 16, torch.float32),
    (3, 200, 1000, 8, torch.bfloat16),
    (1, 129, 512, 3, torch.float32),
    (2, 50, 333, 16, torch.float32),      # a shape the staged kernels do not take
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:4])) + str(c[4])[-4:])
def test_noalloc_matches_regular_forward_on_two_calls(case):
    b, d, L, N, dtype = case
    if (b, d, L, N) == (8, 5120, 2048, 16):
        x = workload_inputs(2, device="cuda", with_dy=False)
    else:
        x = gc.to_device(make_inputs(b, d, L, N, dtype, seed=700 + L))
    y_ref, last_ref = _regular(x)
    tol = gc.TOL[dtype]
    for y, last in _noalloc_twice(x):
        assert torch.isfinite(y.float()).all() and torch.isfinite(last).all()
        ey = gc.normwise(y.cpu().double().numpy(), y_ref.cpu().double().numpy())
        el = gc.normwise(last.cpu().double().numpy(), last_ref.cpu().double().numpy())
        assert ey <= tol and el <= tol, f"y err {ey:.2e}, last_state err {el:.2e}"


def test_noalloc_rejects_problems_beyond_the_array():
    """1024 channel groups of N = 16 need more than the fixed scratch holds
    even for the sequential hand-off: the call is refused on the host and
    nothing is written (the scratch-free one-thread-per-channel kernel is
    10-50 times slower, and a caller who sized for the fast path should
    learn that its problem is beyond it)."""
    x = gc.to_device(make_inputs(8, 16384, 8, 16, torch.bfloat16, seed=9))
    y = torch.zeros_like(x["u"])
    with pytest.raises(scan.MambaScanError) as e:
        scan.mamba_scan_fwd_noalloc(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                    x["D"], x["z"], y, None)
    assert e.value.status == 2  # MAMBA_ERR_UNSUPPORTED
    assert scan.mamba_scan_stream_status() == 0
    assert torch.count_nonzero(y) == 0
