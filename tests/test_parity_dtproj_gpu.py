"""GPU parity of the low-rank Delta projection (mamba_dtproj_scan_fwd / _bwd):
delta = W_dt . dt_low on the tensor cores, then the scan, against the fp64
oracle on the same seeded inputs.  Normwise max error <= 1e-4 for fp32 I/O
and <= 2e-2 for bf16 I/O."""
import math

import pytest
import torch

import gpu_cases as gc
import oracle
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import WORKLOADS, make_inputs, make_dtproj_params

pytestmark = pytest.mark.gpu

GRADS = ("du", "d_dt_low", "dW_dt", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()


def case(b, d, L, N, R, dtype, seed, **kw):
    x = make_inputs(b, d, L, N, dtype, seed=seed, with_dy=True, **kw)
    x.update(make_dtproj_params(b, d, L, R, dtype, seed=seed))
    return x


def gpu_fwd(x, **kw):
    batch, dim, L = x["u"].shape
    y = torch.empty_like(x["u"])
    last = torch.empty(batch, dim, x["A"].shape[1], device="cuda")
    scan.mamba_dtproj_scan_fwd(x["u"], x["dt_low"], x["W_dt"], x["delta_bias"], x["A"], x["B"],
                               x["C"], x["D"], x["z"], y, last, **kw)
    assert scan.mamba_scan_stream_status() == 0
    return y, last


def gpu_bwd(x, **kw):
    dim, N = x["A"].shape
    f32 = dict(device="cuda", dtype=torch.float32)
    g = {"du": torch.empty_like(x["u"]), "d_dt_low": torch.empty_like(x["dt_low"]),
         "dW_dt": torch.empty(x["W_dt"].shape, **f32), "dA": torch.empty(dim, N, **f32),
         "dB": torch.empty_like(x["B"]), "dC": torch.empty_like(x["C"]),
         "dD": torch.empty(dim, **f32) if x["D"] is not None else None,
         "dz": torch.empty_like(x["u"]) if x["z"] is not None else None,
         "ddelta_bias": torch.empty(dim, **f32)}
    scan.mamba_dtproj_scan_bwd(x["u"], x["dt_low"], x["W_dt"], x["delta_bias"], x["A"], x["B"],
                               x["C"], x["D"], x["z"], x["dy"], g["du"], g["d_dt_low"],
                               g["dW_dt"], g["dA"], g["dB"], g["dC"], g["dD"], g["dz"],
                               g["ddelta_bias"], **kw)
    assert scan.mamba_scan_stream_status() == 0
    return {k: v for k, v in g.items() if v is not None}


def oracle_fwd(x):
    return oracle.s6_dtproj_forward(x["u"], x["dt_low"], x["W_dt"], x["A"], x["B"], x["C"],
                                    x["delta_bias"], x["D"], x["z"])


def oracle_bwd(x):
    return oracle.s6_dtproj_backward(x["u"], x["dt_low"], x["W_dt"], x["A"], x["B"], x["C"],
                                     x["dy"], x["delta_bias"], x["D"], x["z"])


def check(xh, fwd=True, bwd=True, **kw):
    x = gc.to_device(xh)
    tol = gc.TOL[xh["u"].dtype]
    if fwd:
        y, last = gpu_fwd(x, **kw)
        y_ref, last_ref = oracle_fwd(xh)
        ey = gc.normwise(y.cpu().double().numpy(), y_ref)
        el = gc.normwise(last.cpu().double().numpy(), last_ref)
        assert ey <= tol and el <= max(tol, 1e-4), f"y err {ey:.2e}, last_state err {el:.2e}"
    if bwd:
        g = gpu_bwd(x, **kw)
        ref = oracle_bwd(xh)
        errs = {k: gc.normwise(g[k].cpu().double().numpy(), ref[k]) for k in GRADS if k in g}
        assert set(errs) == {k for k in GRADS if k in ref}
        bad = {k: v for k, v in errs.items() if not v <= tol}
        assert not bad, f"gradient errors above {tol}: {bad} (all: {errs})"


# (batch, dim, L, N, R): staged scan shapes (ragged channel groups, several
# tiles), a one-thread-per-channel shape, and the rank-1 projection that the
# pages give as the default (one scalar per token broadcast over channels)
SHAPES = [(2, 300, 1056, 16, 20), (1, 130, 512, 8, 8), (2, 37, 50, 4, 5), (2, 200, 256, 16, 1)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_dtproj_grid(shape, dtype):
    b, d, L, N, R = shape
    check(case(b, d, L, N, R, dtype, seed=1100 + L + R))


def test_dtproj_without_gate_and_skip():
    x = case(2, 96, 320, 16, 12, torch.float32, seed=1190, has_z=False, has_D=False)
    x["delta_bias"] = None
    check(x)


def test_dtproj_chunked_paths():
    x = case(1, 130, 1024, 16, 16, torch.float32, seed=1191)
    check(x, chunk_len=192)
    check(x, bwd=False, chunk_len=192, carry="three_phase")


def test_dtproj_bwd_deterministic():
    x = gc.to_device(case(2, 300, 1024, 16, 40, torch.bfloat16, seed=1192))
    g1, g2 = gpu_bwd(x), gpu_bwd(x)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_dtproj_matches_plain_scan_of_projected_delta():
    """The GPU projection is a plain product: the scan of the same delta made
    by torch gives the same y."""
    x = gc.to_device(case(2, 256, 512, 16, 16, torch.float32, seed=1193))
    y, last = gpu_fwd(x)
    delta = torch.matmul(x["W_dt"], x["dt_low"])
    y2, last2 = scan.selective_scan_fwd(x["u"], delta, x["A"], x["B"], x["C"], D=x["D"],
                                        z=x["z"], delta_bias=x["delta_bias"],
                                        return_last_state=True)
    assert gc.normwise(y.cpu().numpy(), y2.cpu().numpy()) <= 1e-4
    assert gc.normwise(last.cpu().numpy(), last2.cpu().numpy()) <= 1e-4


def test_dtproj_full_size_sampled():
    """The bf16 8 x 5120 x 2048 workload with a rank-160 projection (d_model
    2560 / 16): y, du and dz on sampled channels; d_dt_low (a sum over all
    channels) on one whole batch row; dW_dt and dA on a few channels (sums
    over the batch)."""
    w = WORKLOADS[2]
    R = math.ceil(w.dim / 2 / 16)
    xh = case(w.batch, w.dim, w.L, w.N, R, w.dtype, seed=1194)
    x = gc.to_device(xh)
    y, _ = gpu_fwd(x)
    g = gpu_bwd(x)
    tol = gc.TOL[w.dtype]
    yh, gh = y.cpu(), {k: v.cpu() for k, v in g.items()}
    per_d = lambda t, idx: None if t is None else t.index_select(0, idx).contiguous()
    for b, ds in gc.sample_channels(w.batch, w.dim, 8, seed=3).items():
        idx = torch.tensor(ds)
        sub = {k: (None if v is None else v[b:b + 1].index_select(1, idx).contiguous())
               for k, v in xh.items() if k in ("u", "z", "dy")}
        sub.update(B=xh["B"][b:b + 1].contiguous(), C=xh["C"][b:b + 1].contiguous(),
                   A=per_d(xh["A"], idx), D=per_d(xh["D"], idx),
                   delta_bias=per_d(xh["delta_bias"], idx), W_dt=per_d(xh["W_dt"], idx),
                   dt_low=xh["dt_low"][b:b + 1].contiguous())
        y_ref, _ = oracle_fwd(sub)
        e = gc.normwise(yh[b].index_select(0, idx).double().numpy(), y_ref[0])
        assert e <= tol, f"y (batch {b}): {e:.2e}"
        ref = oracle_bwd(sub)
        for k in ("du", "dz"):
            e = gc.normwise(gh[k][b].index_select(0, idx).double().numpy(), ref[k][0])
            assert e <= tol, f"{k} (batch {b}): {e:.2e}"
    b = w.batch - 1
    row = {k: (None if xh[k] is None else xh[k][b:b + 1].contiguous())
           for k in ("u", "z", "dy", "B", "C", "dt_low")}
    row.update(A=xh["A"], D=xh["D"], delta_bias=xh["delta_bias"], W_dt=xh["W_dt"])
    e = gc.normwise(gh["d_dt_low"][b].double().numpy(), oracle_bwd(row)["d_dt_low"][0])
    assert e <= tol, f"d_dt_low (batch {b}): {e:.2e}"
    ds = [0, 4095, w.dim - 1]
    idx = torch.tensor(ds)
    sub = {k: xh[k].index_select(1, idx).contiguous() for k in ("u", "z", "dy")}
    sub.update(B=xh["B"], C=xh["C"], A=per_d(xh["A"], idx), D=per_d(xh["D"], idx),
               delta_bias=per_d(xh["delta_bias"], idx), W_dt=per_d(xh["W_dt"], idx),
               dt_low=xh["dt_low"])
    ref = oracle_bwd(sub)
    for k in ("dW_dt", "dA"):
        e = gc.normwise(gh[k].index_select(0, idx).double().numpy(), ref[k])
        assert e <= tol, f"{k}: {e:.2e}"


@pytest.mark.parametrize("shape", [(2, 24, 1, 4, 3), (1, 16, 64, 8, 40)],
                         ids=lambda s: "x".join(map(str, s)))
def test_dtproj_edge_shapes(shape):
    """A single step, and a rank above dim."""
    b, d, L, N, R = shape
    check(case(b, d, L, N, R, torch.float32, seed=1195 + L + R))


# ---- the training pair: mamba_dtproj_scan_fwd_save / _bwd_saved ----------

def gpu_pair(x, **kw):
    """The saving forward, then the backward reading what it stored."""
    batch, dim, L = x["u"].shape
    N, R = x["A"].shape[1], x["W_dt"].shape[1]
    need = scan.dtproj_saved_bytes(batch, dim, L, N, R, x["u"].dtype, **kw)
    saved = torch.empty(max(need, 1), device="cuda", dtype=torch.uint8) if need else None
    y = torch.empty_like(x["u"])
    last = torch.empty(batch, dim, N, device="cuda")
    scan.mamba_dtproj_scan_fwd_save(x["u"], x["dt_low"], x["W_dt"], x["delta_bias"], x["A"],
                                    x["B"], x["C"], x["D"], x["z"], y, last, saved, **kw)
    f32 = dict(device="cuda", dtype=torch.float32)
    g = {"du": torch.empty_like(x["u"]), "d_dt_low": torch.empty_like(x["dt_low"]),
         "dW_dt": torch.empty(x["W_dt"].shape, **f32), "dA": torch.empty(dim, N, **f32),
         "dB": torch.empty_like(x["B"]), "dC": torch.empty_like(x["C"]),
         "dD": torch.empty(dim, **f32) if x["D"] is not None else None,
         "dz": torch.empty_like(x["u"]) if x["z"] is not None else None,
         "ddelta_bias": torch.empty(dim, **f32)}
    scan.mamba_dtproj_scan_bwd_saved(x["u"], x["dt_low"], x["W_dt"], x["delta_bias"], x["A"],
                                     x["B"], x["C"], x["D"], x["z"], x["dy"], g["du"],
                                     g["d_dt_low"], g["dW_dt"], g["dA"], g["dB"], g["dC"],
                                     g["dD"], g["dz"], g["ddelta_bias"], saved, **kw)
    assert scan.mamba_scan_stream_status() == 0
    return need, y, last, {k: v for k, v in g.items() if v is not None}


def _close(a, b, bound, what):
    e = gc.normwise(a.cpu().double().numpy(), b.cpu().double().numpy())
    assert e <= bound, f"{what}: pair vs plain {e:.2e}"


# L <= 256 puts the backward in one chunk, carried in sequence, whatever the
# grid: the fused pair stores states on these shapes
PAIR_SHAPES = [(2, 200, 256, 16, 1), (2, 300, 256, 16, 20), (1, 130, 128, 8, 8),
               (3, 64, 200, 4, 5)]


@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_dtproj_pair_against_oracle_and_plain(shape):
    b, d, L, N, R = shape
    xh = case(b, d, L, N, R, torch.bfloat16, seed=1300 + L + R)
    x = gc.to_device(xh)
    need, y, last, g = gpu_pair(x)
    assert need > 0
    tol = gc.TOL[torch.bfloat16]
    y_ref, last_ref = oracle_fwd(xh)
    assert gc.normwise(y.cpu().double().numpy(), y_ref) <= tol
    assert gc.normwise(last.cpu().double().numpy(), last_ref) <= 1e-4
    ref = oracle_bwd(xh)
    errs = {k: gc.normwise(g[k].cpu().double().numpy(), ref[k]) for k in GRADS if k in g}
    assert all(v <= tol for v in errs.values()), errs
    # the same arithmetic as the recomputing calls, to rounding
    y0, last0 = gpu_fwd(x)
    g0 = gpu_bwd(x)
    _close(y, y0, 1e-4, "y")
    _close(last, last0, 1e-6, "last_state")
    for k in g0:
        _close(g[k], g0[k], 1e-4, k)


def test_dtproj_pair_without_gate_skip_and_bias():
    xh = case(2, 96, 256, 16, 12, torch.bfloat16, seed=1310, has_z=False, has_D=False)
    xh["delta_bias"] = None
    x = gc.to_device(xh)
    need, y, _, g = gpu_pair(x)
    assert need > 0
    tol = gc.TOL[torch.bfloat16]
    assert gc.normwise(y.cpu().double().numpy(), oracle_fwd(xh)[0]) <= tol
    ref = oracle_bwd(xh)
    for k in g:
        assert gc.normwise(g[k].cpu().double().numpy(), ref[k]) <= tol, k


def test_dtproj_pair_stores_nothing_where_the_backward_splits_the_sequence():
    """A short batch of long rows: the backward carries its adjoint through
    three phases, so the pair stores nothing and behaves as the plain calls
    (also for fp32, which the fused kernels do not take)."""
    for dtype in (torch.bfloat16, torch.float32):
        xh = case(1, 130, 1024, 16, 16, dtype, seed=1311)
        x = gc.to_device(xh)
        need, y, last, g = gpu_pair(x)
        assert need == 0
        y0, last0 = gpu_fwd(x)
        g0 = gpu_bwd(x)
        assert torch.equal(y, y0) and torch.equal(last, last0)
        for k in g0:
            assert torch.equal(g[k], g0[k]), k


def test_dtproj_pair_refusals():
    """A buffer shorter than dtproj_saved_bytes, and a dt_low off the 16-byte
    grid (which the fused kernels cannot read with their tensor maps), are
    refused before anything is enqueued."""
    x = gc.to_device(case(2, 200, 256, 16, 8, torch.bfloat16, seed=1312))
    need = scan.dtproj_saved_bytes(2, 200, 256, 16, 8, torch.bfloat16)
    assert need > 0
    y = torch.empty_like(x["u"])
    short = torch.empty(need - 16, device="cuda", dtype=torch.uint8)
    with pytest.raises(ValueError):
        scan.mamba_dtproj_scan_fwd_save(x["u"], x["dt_low"], x["W_dt"], x["delta_bias"], x["A"],
                                        x["B"], x["C"], x["D"], x["z"], y, None, short)
    base = torch.empty(x["dt_low"].numel() + 1, device="cuda", dtype=torch.bfloat16)
    odd = base[1:].view_as(x["dt_low"])
    odd.copy_(x["dt_low"])
    saved = torch.empty(need, device="cuda", dtype=torch.uint8)
    launches0 = scan.launch_count()
    with pytest.raises(scan.MambaScanError) as e:
        scan.mamba_dtproj_scan_fwd_save(x["u"], odd, x["W_dt"], x["delta_bias"], x["A"], x["B"],
                                        x["C"], x["D"], x["z"], y, None, saved)
    assert e.value.status == 1  # MAMBA_ERR_INVALID_ARG
    assert scan.launch_count() == launches0
    assert scan.mamba_scan_stream_status() == 0


def test_dtproj_pair_full_size():
    """The bf16 8 x 5120 x 2048 workload with the rank-160 projection: the
    pair stores states and agrees with the recomputing calls; y and du on
    sampled channels against the oracle."""
    w = WORKLOADS[2]
    R = math.ceil(w.dim / 2 / 16)
    xh = case(w.batch, w.dim, w.L, w.N, R, w.dtype, seed=1194)
    x = gc.to_device(xh)
    need, y, _, g = gpu_pair(x)
    assert need > 0
    y0, _ = gpu_fwd(x)
    g0 = gpu_bwd(x)
    _close(y, y0, 1e-4, "y")
    for k in g0:
        _close(g[k], g0[k], 1e-3, k)
    tol = gc.TOL[w.dtype]
    per_d = lambda t, idx: None if t is None else t.index_select(0, idx).contiguous()
    for b, ds in gc.sample_channels(w.batch, w.dim, 4, seed=5).items():
        idx = torch.tensor(ds)
        sub = {k: (None if v is None else v[b:b + 1].index_select(1, idx).contiguous())
               for k, v in xh.items() if k in ("u", "z", "dy")}
        sub.update(B=xh["B"][b:b + 1].contiguous(), C=xh["C"][b:b + 1].contiguous(),
                   A=per_d(xh["A"], idx), D=per_d(xh["D"], idx),
                   delta_bias=per_d(xh["delta_bias"], idx), W_dt=per_d(xh["W_dt"], idx),
                   dt_low=xh["dt_low"][b:b + 1].contiguous())
        e = gc.normwise(y[b].cpu().index_select(0, idx).double().numpy(), oracle_fwd(sub)[0][0])
        assert e <= tol, f"y (batch {b}): {e:.2e}"
        e = gc.normwise(g["du"][b].cpu().index_select(0, idx).double().numpy(),
                        oracle_bwd(sub)["du"][0])
        assert e <= tol, f"du (batch {b}): {e:.2e}"
