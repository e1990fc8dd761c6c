"""The training pair (mamba_scan_fwd_save / mamba_scan_bwd_saved): the forward
stores the states the backward would recompute, the backward reads them.
Its y and gradients must match mamba_scan_fwd's and mamba_scan_bwd's (same
formulas on the same chunking: bit for bit where the kernels compile them
alike, which the bf16 cases and the fp32 three-phase gradients show; within
1e-5 normwise otherwise, the saving kernel being a different instance whose
FMA contractions may differ), and both must match the fp64 oracle."""
import pytest
import torch

import gpu_cases as gc
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

GRAD_KEYS = ["du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()


def _pair(x, **opts):
    y, last, saved = scan.selective_scan_fwd_save(x["u"], x["delta"], x["A"], x["B"], x["C"],
                                                  D=x["D"], z=x["z"], delta_bias=x["delta_bias"],
                                                  return_last_state=True, **opts)
    g = scan.selective_scan_bwd_saved(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"], saved,
                                      D=x["D"], z=x["z"], delta_bias=x["delta_bias"], **opts)
    assert scan.mamba_scan_stream_status() == 0
    return y, last, saved, g


def _plain(x, **opts):
    y, last = gc.gpu_fwd(x, **opts)
    return y, last, gc.gpu_bwd(x, **opts)


def _close(a, b, tol):
    return gc.normwise(a.cpu().double().numpy(), b.cpu().double().numpy()) <= tol


def _check_pair(x_host, y_exact=True, g_exact=True, oracle=True, **opts):
    x = gc.to_device(x_host)
    y, last, saved, g = _pair(x, **opts)
    y0, last0, g0 = _plain(x, **opts)
    if y_exact:
        assert torch.equal(y, y0) and torch.equal(last, last0)
    else:
        tol = gc.TOL[x_host["u"].dtype]
        assert _close(y, y0, tol) and _close(last, last0, 1e-5)
    for k in GRAD_KEYS:
        if k in g0:
            if g_exact:
                assert torch.equal(g[k], g0[k]), f"{k} differs from the recomputing backward"
            else:  # fp32: rounding of the states; bf16: that can flip an output's last bit
                gt = 1e-5 if x_host["u"].dtype == torch.float32 else gc.TOL[x_host["u"].dtype]
                assert _close(g[k], g0[k], gt), f"{k} differs from the recomputing backward"
    if oracle:
        ref = gc.oracle_bwd(x_host)
        tol = gc.TOL[x_host["u"].dtype]
        errs = {k: gc.normwise(g[k].cpu().double().numpy(), ref[k]) for k in GRAD_KEYS
                if k in g and k in ref}
        assert all(e <= tol for e in errs.values()), errs
        y_ref, _ = gc.oracle_fwd(x_host)
        assert gc.normwise(y.cpu().double().numpy(), y_ref) <= tol
    return saved


# (batch, dim, L, N): few channel groups (three-phase chunks from zero,
# ragged L) and enough groups to fill the GPU (sequential hand-off)
THREE_PHASE = [(2, 256, 2048, 16), (1, 200, 1000, 8), (2, 130, 1536, 4)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", THREE_PHASE, ids=lambda s: "x".join(map(str, s)))
def test_pair_three_phase(shape, dtype):
    b, d, L, N = shape
    x = make_inputs(b, d, L, N, dtype, seed=700 + L, with_dy=True)
    # bf16: the same zero-start chunks and correction on both sides, bit for
    # bit; fp32: the saving forward stores the true states (aggregate pass),
    # the recomputing backward corrects zero-start checkpoints: to rounding
    exact = dtype == torch.bfloat16
    saved = _check_pair(x, y_exact=exact, g_exact=exact)
    assert saved is not None and saved.numel() == scan.saved_bytes(b, d, L, N, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_pair_sequential_handoff(dtype):
    """40 groups of 128 channels per batch row x 8 rows fill the GPU: the
    forward's chunks (four of 256 steps) hand their states on in sequence."""
    x = make_inputs(8, 5120, 1024, 16, dtype, seed=710, with_dy=True)
    exact = dtype == torch.bfloat16
    _check_pair(x, y_exact=exact, g_exact=exact, oracle=False)


def test_pair_generic_A_and_generic_path():
    x = make_inputs(2, 96, 640, 16, torch.bfloat16, seed=720, with_dy=True)
    x["A"] = -torch.exp(torch.randn(96, 16, generator=torch.Generator().manual_seed(3)) * 0.5)
    _check_pair(x)
    _check_pair(make_inputs(2, 96, 640, 16, torch.bfloat16, seed=721, with_dy=True), path="generic")


@pytest.mark.parametrize("has_z,has_D", [(False, False), (True, False), (False, True)])
def test_pair_optional_inputs(has_z, has_D):
    x = make_inputs(2, 160, 512, 16, torch.float32, seed=730, has_z=has_z, has_D=has_D,
                    with_dy=True)
    _check_pair(x, y_exact=False, g_exact=False)


def test_pair_saved_serves_two_backwards():
    x = gc.to_device(make_inputs(2, 128, 1024, 16, torch.bfloat16, seed=740, with_dy=True))
    _, _, saved, g1 = _pair(x)
    g2 = scan.selective_scan_bwd_saved(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"], saved,
                                       D=x["D"], z=x["z"], delta_bias=x["delta_bias"])
    for k in g1:
        assert torch.equal(g1[k], g2[k])


def test_pair_without_saved_states():
    """N = 2 and the reference path save nothing: the pair is the plain calls."""
    x = gc.to_device(make_inputs(2, 64, 300, 2, torch.float32, seed=750, with_dy=True))
    assert scan.saved_bytes(2, 64, 300, 2, torch.float32) == 0
    y, last, saved, g = _pair(x)
    assert saved is None
    y0, last0, g0 = _plain(x)
    assert torch.equal(y, y0)
    for k in g0:
        assert torch.equal(g[k], g0[k])
    assert scan.saved_bytes(2, 64, 512, 16, torch.float32, path="reference") == 0


def test_pair_refuses_a_short_buffer():
    x = gc.to_device(make_inputs(1, 128, 512, 16, torch.bfloat16, seed=760))
    need = scan.saved_bytes(1, 128, 512, 16, torch.bfloat16)
    assert need > 0
    short = torch.empty(need - 256, device="cuda", dtype=torch.uint8)
    y = torch.empty_like(x["u"])
    with pytest.raises(ValueError):
        scan.mamba_scan_fwd_save(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                 x["D"], x["z"], y, None, short)
    # the C entry point itself refuses it too (nothing enqueued)
    import ctypes
    lib = scan.load_library()
    rc = lib.mamba_scan_fwd_save(
        x["u"].data_ptr(), x["delta"].data_ptr(), x["delta_bias"].data_ptr(), x["A"].data_ptr(),
        x["B"].data_ptr(), x["C"].data_ptr(), x["D"].data_ptr(), x["z"].data_ptr(), y.data_ptr(),
        None, 1, 128, 512, 16, scan._dtype_code(torch.bfloat16), None, short.data_ptr(),
        ctypes.c_uint64(short.numel()), None)
    assert rc == 1  # MAMBA_ERR_INVALID_ARG


def test_pair_full_bench_workload():
    """bf16 8 x 5120 x 2048 (the benchmark's step, in its launch configuration):
    the pair's y and gradients equal the plain calls' bit for bit, which the
    full-size sampled oracle tests check against the fp64 oracle."""
    x = workload_inputs(2, device="cuda", with_dy=True)
    y, last, saved, g = _pair(x)
    y0, last0, g0 = _plain(x)
    assert torch.equal(y, y0) and torch.equal(last, last0)
    for k in g0:
        assert torch.equal(g[k], g0[k]), k


# ------------------------------------------------ with the convolution prologue

CONV_GRADS = ("dx", "dconv_w", "dconv_b", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")


def _conv_case(b, d, L, N, dtype, W=4, seed=0):
    from selective_state_space_21_b200.inputs import make_conv_params
    x = make_inputs(b, d, L, N, dtype, seed=seed, with_dy=True)
    x.update(make_conv_params(d, W, seed=seed, has_bias=True))
    return x


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 256, 2048, 16), (8, 5120, 512, 16)],
                         ids=["three_phase", "sequential"])
def test_conv_pair(shape, dtype):
    """mamba_conv_scan_fwd_save / _bwd_saved against the plain conv calls (bit
    for bit in bf16) and, at the small shape, the fp64 conv oracle."""
    import oracle
    b, d, L, N = shape
    xh = _conv_case(b, d, L, N, dtype, seed=800 + b)
    x = gc.to_device(xh)
    kw = dict(D=x["D"], z=x["z"], delta_bias=x["delta_bias"])
    y, last, saved = scan.conv_selective_scan_fwd_save(x["u"], x["conv_w"], x["conv_b"],
                                                       x["delta"], x["A"], x["B"], x["C"],
                                                       return_last_state=True, **kw)
    g = scan.conv_selective_scan_bwd_saved(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"],
                                           x["B"], x["C"], x["dy"], saved, **kw)
    y0, last0 = scan.conv_selective_scan_fwd(x["u"], x["conv_w"], x["conv_b"], x["delta"],
                                             x["A"], x["B"], x["C"], return_last_state=True, **kw)
    g0 = scan.conv_selective_scan_bwd(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"],
                                      x["B"], x["C"], x["dy"], **kw)
    assert scan.mamba_scan_stream_status() == 0
    assert saved is not None
    exact = dtype == torch.bfloat16
    tol = gc.TOL[dtype]
    if exact:
        assert torch.equal(y, y0) and torch.equal(last, last0)
    else:
        assert _close(y, y0, tol) and _close(last, last0, 1e-5)
    for k in CONV_GRADS:
        if k in g0:
            assert torch.equal(g[k], g0[k]) if exact else _close(g[k], g0[k], 1e-5), k
    if b == 2:
        ref = oracle.s6_conv_backward(xh["u"], xh["conv_w"], xh["conv_b"], xh["delta"], xh["A"],
                                      xh["B"], xh["C"], xh["dy"], xh["delta_bias"], xh["D"],
                                      xh["z"])
        errs = {k: gc.normwise(g[k].cpu().double().numpy(), ref[k]) for k in CONV_GRADS
                if k in g and k in ref}
        assert all(e <= tol for e in errs.values()), errs


@pytest.mark.parametrize("carry,chunk_len", [("sequential", 256), ("three_phase", 192),
                                             ("three_phase", 0)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_pair_explicit_chunking(carry, chunk_len, dtype):
    """Explicit chunking options reach the saving forward and the backward
    alike (the saved layout follows them): the gradients match the fp64
    oracle and, within rounding, the recomputing backward (whose own forward
    pass takes the automatic chunking)."""
    xh = make_inputs(2, 160, 1100, 16, dtype, seed=900 + chunk_len, with_dy=True)
    _check_pair(xh, y_exact=False, g_exact=False, carry=carry, chunk_len=chunk_len)
