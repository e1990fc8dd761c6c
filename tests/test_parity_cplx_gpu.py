"""GPU parity of the complex-A scan (mamba_cplx_scan_fwd / _bwd, S4D-Lin
A_n = -1/2 + n i, complex B and C) against the fp64 oracle on the same seeded
inputs.  Normwise max error <= 1e-4 for fp32 I/O and <= 2e-2 for bf16 I/O."""
import numpy as np
import pytest
import torch

import gpu_cases as gc
import oracle
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import WORKLOADS, make_cplx_inputs, make_inputs

pytestmark = pytest.mark.gpu

GRADS = ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()


def gpu_fwd(x):
    batch, dim, L = x["u"].shape
    y = torch.empty_like(x["u"])
    last = torch.empty(batch, dim, x["A"].shape[1], device="cuda")
    scan.mamba_cplx_scan_fwd(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"],
                             x["z"], y, last)
    assert scan.mamba_scan_stream_status() == 0
    return y, last


def gpu_bwd(x):
    dim, N2 = x["A"].shape
    f32 = dict(device="cuda", dtype=torch.float32)
    g = {"du": torch.empty_like(x["u"]), "ddelta": torch.empty_like(x["u"]),
         "dA": torch.empty(dim, N2, **f32), "dB": torch.empty_like(x["B"]),
         "dC": torch.empty_like(x["C"]),
         "dD": torch.empty(dim, **f32) if x["D"] is not None else None,
         "dz": torch.empty_like(x["u"]) if x["z"] is not None else None,
         "ddelta_bias": torch.empty(dim, **f32)}
    scan.mamba_cplx_scan_bwd(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"],
                             x["z"], x["dy"], g["du"], g["ddelta"], g["dA"], g["dB"], g["dC"],
                             g["dD"], g["dz"], g["ddelta_bias"])
    assert scan.mamba_scan_stream_status() == 0
    return {k: v for k, v in g.items() if v is not None}


def check(xh, fwd=True, bwd=True):
    x = gc.to_device(xh)
    tol = gc.TOL[xh["u"].dtype]
    args = (xh["u"], xh["delta"], xh["A"], xh["B"], xh["C"])
    kw = dict(delta_bias=xh["delta_bias"], D=xh["D"], z=xh["z"])
    if fwd:
        y, last = gpu_fwd(x)
        y_ref, last_ref = oracle.s6_cplx_forward(*args, **kw)
        ey = gc.normwise(y.cpu().double().numpy(), y_ref)
        el = gc.normwise(last.cpu().double().numpy(), last_ref)
        assert ey <= tol and el <= max(tol, 1e-4), f"y err {ey:.2e}, last_state err {el:.2e}"
    if bwd:
        g = gpu_bwd(x)
        ref = oracle.s6_cplx_backward(*args, xh["dy"], **kw)
        errs = {k: gc.normwise(g[k].cpu().double().numpy(), ref[k]) for k in GRADS if k in g}
        assert set(errs) == {k for k in GRADS if k in ref}
        bad = {k: v for k, v in errs.items() if not v <= tol}
        assert not bad, f"gradient errors above {tol}: {bad} (all: {errs})"


# N = 12 and 5 leave whole threads of a channel with padding states only
SHAPES = [(2, 200, 300, 16), (1, 70, 129, 8), (3, 5, 40, 1), (2, 130, 77, 4), (1, 33, 20, 3),
          (2, 50, 33, 12), (1, 40, 17, 5), (1, 9, 1, 16)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_cplx_grid(shape, dtype):
    b, d, L, N = shape
    check(make_cplx_inputs(b, d, L, N, dtype, seed=1300 + L + d, with_dy=True))


def test_cplx_without_gate_and_skip():
    x = make_cplx_inputs(2, 96, 100, 16, torch.float32, seed=1390, has_z=False, has_D=False,
                         with_dy=True)
    x["delta_bias"] = None
    check(x)


def test_cplx_random_complex_A():
    """A with random negative real parts and imaginary parts of either sign
    (not the S4D-Lin pattern), including small |Delta A| where psi and phi
    take their series."""
    x = make_cplx_inputs(2, 64, 90, 8, torch.float32, seed=1391, with_dy=True)
    g = torch.Generator().manual_seed(9)
    re = -torch.exp(torch.randn(64, 8, generator=g) * 1.5)
    im = torch.randn(64, 8, generator=g) * 3.0
    re[0, :2] = -1e-4
    im[0, :2] = 0.0
    x["A"] = torch.cat([re, im], dim=1).contiguous()
    check(x)


def test_cplx_mixed_structure_and_large_angles():
    """A_n = a + i s (n - 5): evenly spaced imaginary parts that change sign
    inside some threads' groups of states (those take the per-state decay, the
    rest the shared half-angle recurrence), spacings s up to 8 so that one
    step turns a state by up to some twenty full circles, a real part per
    channel, and channels whose spacing is not exact in fp32 next to ones
    whose is.  Channels 3 and 11 have evenly spaced A with |A| below 1/8 in
    their first states (the structured decay without the h += M (h + B u/A)
    update).  (Much larger |Delta A| leaves fp32 short of the 1e-4 bound on
    ddelta whichever decay runs: dA/dDelta carries the factor A.)"""
    dim, N = 96, 16
    x = make_cplx_inputs(2, dim, 150, N, torch.float32, seed=1394, with_dy=True)
    n = torch.arange(N, dtype=torch.float32)
    s = (torch.arange(dim) % 8 + 1).float()
    s[1::2] += 0.1
    re = -torch.linspace(0.05, 3.0, dim)[:, None].expand(dim, N).clone()
    im = (n - 5.0)[None, :] * s[:, None]
    for d in (3, 11):
        re[d] = -0.06
        im[d] = 0.01 * n
    x["A"] = torch.cat([re, im], dim=1).contiguous()
    check(x)


def test_cplx_real_case_matches_real_scan():
    """Zero imaginary parts: the complex kernels give the real kernels' y and
    gradients."""
    xr = gc.to_device(make_inputs(2, 150, 256, 8, torch.float32, seed=1392, with_dy=True))
    z2 = lambda t: torch.cat([t, torch.zeros_like(t)], dim=1).contiguous()
    xc = dict(xr, A=z2(xr["A"]), B=z2(xr["B"]), C=z2(xr["C"]))
    y, last = gpu_fwd(xc)
    y_r, last_r = gc.gpu_fwd(xr, path="reference")
    assert gc.normwise(y.cpu().numpy(), y_r.cpu().numpy()) <= 1e-5
    assert gc.normwise(last[..., :8].cpu().numpy(), last_r.cpu().numpy()) <= 1e-5
    g = gpu_bwd(xc)
    gr = gc.gpu_bwd(xr, path="reference")
    for k in ("du", "ddelta", "dz", "dD", "ddelta_bias"):
        assert gc.normwise(g[k].cpu().numpy(), gr[k].cpu().numpy()) <= 1e-4, k
    assert gc.normwise(g["dA"][:, :8].cpu().numpy(), gr["dA"].cpu().numpy()) <= 1e-4
    for k in ("dB", "dC"):
        assert gc.normwise(g[k][:, :8].cpu().numpy(), gr[k].cpu().numpy()) <= 1e-4, k


def test_cplx_bwd_deterministic():
    x = gc.to_device(make_cplx_inputs(2, 300, 200, 16, torch.bfloat16, seed=1393, with_dy=True))
    g1, g2 = gpu_bwd(x), gpu_bwd(x)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


@pytest.mark.parametrize("wl", [2, 4], ids=["b8_d5120_L2048", "b4_d2048_L4096"])
def test_cplx_full_size_sampled(wl):
    """Workload shapes with 16 complex states (bf16 8 x 5120 x 2048, the one
    the bench times, and 4 x 2048 x 4096): y, du, ddelta and dz on sampled
    channels against the oracle, and dA, dD, dbias (sums over the batch) on
    three channels."""
    w = WORKLOADS[wl]
    xh = make_cplx_inputs(w.batch, w.dim, w.L, w.N, w.dtype, seed=1394 + wl, with_dy=True)
    x = gc.to_device(xh)
    y, _ = gpu_fwd(x)
    g = gpu_bwd(x)
    tol = gc.TOL[w.dtype]
    yh, gh = y.cpu(), {k: v.cpu() for k, v in g.items()}
    per_d = lambda t, idx: None if t is None else t.index_select(0, idx).contiguous()
    for b, ds in gc.sample_channels(w.batch, w.dim, 8, seed=4).items():
        idx = torch.tensor(ds)
        sub = {k: (None if xh[k] is None else xh[k][b:b + 1].index_select(1, idx).contiguous())
               for k in ("u", "delta", "z", "dy")}
        sub.update(B=xh["B"][b:b + 1].contiguous(), C=xh["C"][b:b + 1].contiguous(),
                   A=per_d(xh["A"], idx), D=per_d(xh["D"], idx),
                   delta_bias=per_d(xh["delta_bias"], idx))
        args = (sub["u"], sub["delta"], sub["A"], sub["B"], sub["C"])
        kw = dict(delta_bias=sub["delta_bias"], D=sub["D"], z=sub["z"])
        y_ref, _ = oracle.s6_cplx_forward(*args, **kw)
        e = gc.normwise(yh[b].index_select(0, idx).double().numpy(), y_ref[0])
        assert e <= tol, f"y (batch {b}): {e:.2e}"
        ref = oracle.s6_cplx_backward(*args, sub["dy"], **kw)
        for k in ("du", "ddelta", "dz"):
            e = gc.normwise(gh[k][b].index_select(0, idx).double().numpy(), ref[k][0])
            assert e <= tol, f"{k} (batch {b}): {e:.2e}"
    idx = torch.tensor([0, w.dim // 2 + 1, w.dim - 1])
    sub = {k: xh[k].index_select(1, idx).contiguous() for k in ("u", "delta", "z", "dy")}
    sub.update(A=per_d(xh["A"], idx), D=per_d(xh["D"], idx), delta_bias=per_d(xh["delta_bias"], idx))
    ref = oracle.s6_cplx_backward(sub["u"], sub["delta"], sub["A"], xh["B"], xh["C"], sub["dy"],
                                  delta_bias=sub["delta_bias"], D=sub["D"], z=sub["z"])
    for k in ("dA", "dD", "ddelta_bias"):
        e = gc.normwise(gh[k].index_select(0, idx).double().numpy(), ref[k])
        assert e <= tol, f"{k}: {e:.2e}"


def test_cplx_rejects_bad_arguments():
    """More than 16 complex states is unsupported, and an output over an input
    is an invalid argument.  Nothing is launched for them."""
    x = gc.to_device(make_cplx_inputs(1, 8, 32, 4, torch.float32, seed=1395, with_dy=True))
    y = torch.empty_like(x["u"])
    last = torch.empty(1, 8, 8, device="cuda")
    base = (x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"], x["z"])
    with pytest.raises(scan.MambaScanError) as e:  # y over u
        scan.mamba_cplx_scan_fwd(*base, x["u"], last)
    assert e.value.status == 1  # MAMBA_ERR_INVALID_ARG
    A17 = torch.cat([torch.full((8, 17), -0.5), torch.zeros(8, 17)], dim=1).cuda()
    B17 = torch.zeros(1, 34, 32, device="cuda")
    with pytest.raises(scan.MambaScanError) as e:
        scan.mamba_cplx_scan_fwd(x["u"], x["delta"], x["delta_bias"], A17, B17, B17, x["D"],
                                 x["z"], y, None)
    assert e.value.status == 2  # MAMBA_ERR_UNSUPPORTED
    assert scan.mamba_scan_stream_status() == 0


def test_cplx_bwd_rows_not_16_byte_aligned():
    """Element-aligned tensors that are not 16-byte aligned take the backward's
    per-element block loads and stores instead of the 16-byte ones: the
    gradients are bitwise those of the aligned call."""
    x = gc.to_device(make_cplx_inputs(2, 24, 64, 16, torch.float32, seed=1396, with_dy=True))
    g = gpu_bwd(x)

    def offset(t):  # same values, 4 bytes past a 16-byte boundary
        o = torch.empty(t.numel() + 1, device="cuda", dtype=t.dtype)[1:].view(t.shape)
        o.copy_(t)
        return o

    x2 = dict(x, u=offset(x["u"]), dy=offset(x["dy"]))
    g2 = gpu_bwd(x2)
    for k in g:
        assert torch.equal(g[k], g2[k]), k


def _random_cases(count, seed):
    """Seeded shapes: batch 1-3, dim 1-120, L 1-300 (a multiple of 8 one time
    in two, so that the backward's 16-byte block loads take part), N 1-16."""
    g = np.random.default_rng(seed)
    cases = []
    for i in range(count):
        L = int(g.integers(1, 301))
        if i % 2 == 0:
            L = max(8, L - L % 8)
        cases.append((int(g.integers(1, 4)), int(g.integers(1, 121)), L, int(g.integers(1, 17))))
    return cases


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", _random_cases(8, 2027), ids=lambda s: "x".join(map(str, s)))
def test_cplx_random_shapes(shape, dtype):
    b, d, L, N = shape
    check(make_cplx_inputs(b, d, L, N, dtype, seed=1400 + b * 131 + d + L, with_dy=True))


@pytest.mark.parametrize("shape", [(1, 19040, 40, 16), (2, 9600, 32, 16), (1, 36000, 24, 16),
                                   (1, 38000, 17, 8)], ids=lambda s: "x".join(map(str, s)))
def test_cplx_bwd_many_channels(shape):
    """Channel counts that fill more than half a round of the backward's CTA
    slots, so that it runs four (N = 16) or two (N = 8) threads per channel;
    the smaller shapes above run one state per thread.  Every gradient, dB and
    dC included, against the oracle."""
    b, d, L, N = shape
    check(make_cplx_inputs(b, d, L, N, torch.float32, seed=1500 + d + L, with_dy=True))


def pair(x):
    """The complex training pair: the forward stores the block checkpoints, the
    backward reads them in place of its forward sweep."""
    batch, dim, L = x["u"].shape
    saved = torch.empty(scan.cplx_saved_bytes(batch, dim, L, x["A"].shape[1] // 2, x["u"].dtype),
                        device="cuda", dtype=torch.uint8)
    y = torch.empty_like(x["u"])
    last = torch.empty(batch, dim, x["A"].shape[1], device="cuda")
    scan.mamba_cplx_scan_fwd_save(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                  x["D"], x["z"], y, last, saved)
    dim, N2 = x["A"].shape
    f32 = dict(device="cuda", dtype=torch.float32)
    g = {"du": torch.empty_like(x["u"]), "ddelta": torch.empty_like(x["u"]),
         "dA": torch.empty(dim, N2, **f32), "dB": torch.empty_like(x["B"]),
         "dC": torch.empty_like(x["C"]),
         "dD": torch.empty(dim, **f32) if x["D"] is not None else None,
         "dz": torch.empty_like(x["u"]) if x["z"] is not None else None,
         "ddelta_bias": torch.empty(dim, **f32)}
    scan.mamba_cplx_scan_bwd_saved(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                   x["D"], x["z"], x["dy"], g["du"], g["ddelta"], g["dA"], g["dB"],
                                   g["dC"], g["dD"], g["dz"], g["ddelta_bias"], saved)
    assert scan.mamba_scan_stream_status() == 0
    return y, last, {k: v for k, v in g.items() if v is not None}


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 200, 300, 16), (1, 70, 129, 8), (3, 5, 40, 1),
                                   (1, 9, 1, 16), (2, 50, 33, 12), (8, 2560, 64, 16)],
                         ids=lambda s: "x".join(map(str, s)))
def test_cplx_pair(shape, dtype):
    """y and the gradients of the pair against the plain calls (the same
    recurrence: within 1e-5 normwise in fp32, within the bf16 bar in bf16) and,
    at the small shapes, against the fp64 oracle.  The last shape has more
    channel blocks than CTA slots: four chunks per sequence in the backward."""
    b, d, L, N = shape
    xh = make_cplx_inputs(b, d, L, N, dtype, seed=1600 + d + L, with_dy=True)
    x = gc.to_device(xh)
    y, last, g = pair(x)
    y0, last0 = gpu_fwd(x)
    g0 = gpu_bwd(x)
    assert torch.equal(y, y0) and torch.equal(last, last0)  # the same forward kernel
    gt = 1e-5 if dtype == torch.float32 else gc.TOL[dtype]
    for k in g0:
        if g0[k] is not None:
            e = gc.normwise(g[k].cpu().double().numpy(), g0[k].cpu().double().numpy())
            assert e <= gt, f"{k}: {e:.2e} from the backward with its own forward sweep"
    if b * d * L <= 200 * 300 * 2:
        tol = gc.TOL[dtype]
        kw = dict(delta_bias=xh["delta_bias"], D=xh["D"], z=xh["z"])
        ref = oracle.s6_cplx_backward(xh["u"], xh["delta"], xh["A"], xh["B"], xh["C"], xh["dy"],
                                      **kw)
        errs = {k: gc.normwise(g[k].cpu().double().numpy(), ref[k]) for k in GRADS if k in g}
        assert all(e <= tol for e in errs.values()), errs


def test_cplx_pair_refuses_a_missing_buffer():
    x = gc.to_device(make_cplx_inputs(1, 8, 32, 4, torch.float32, seed=1601, with_dy=True))
    lib = scan.load_library()
    y = torch.empty_like(x["u"])
    rc = lib.mamba_cplx_scan_fwd_save(
        x["u"].data_ptr(), x["delta"].data_ptr(), x["delta_bias"].data_ptr(), x["A"].data_ptr(),
        x["B"].data_ptr(), x["C"].data_ptr(), x["D"].data_ptr(), x["z"].data_ptr(), y.data_ptr(),
        None, 1, 8, 32, 4, scan._dtype_code(torch.float32), None, 0, None)
    assert rc == 1  # MAMBA_ERR_INVALID_ARG
