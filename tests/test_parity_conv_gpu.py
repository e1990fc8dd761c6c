"""GPU parity of the convolution prologue (mamba_conv_scan_fwd / _bwd): the
scan driven by u = SiLU(causal depthwise conv(x)), computed inside the scan
kernels, against the fp64 oracle on the same seeded inputs.  Normwise max
error <= 1e-4 for fp32 I/O and <= 2e-2 for bf16 I/O."""
import pytest
import torch

import gpu_cases as gc
import oracle
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import WORKLOADS, make_conv_params, make_inputs

pytestmark = pytest.mark.gpu

GRADS = ("dx", "dconv_w", "dconv_b", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()


def conv_case(b, d, L, N, dtype, W=4, seed=0, has_bias=True, **kw):
    x = make_inputs(b, d, L, N, dtype, seed=seed, with_dy=True, **kw)
    x.update(make_conv_params(d, W, seed=seed, has_bias=has_bias))
    return x


def gpu_fwd(x, **kw):
    y, last = scan.conv_selective_scan_fwd(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"],
                                           x["B"], x["C"], D=x["D"], z=x["z"],
                                           delta_bias=x["delta_bias"], return_last_state=True,
                                           **kw)
    assert scan.mamba_scan_stream_status() == 0
    return y, last


def gpu_bwd(x, **kw):
    g = scan.conv_selective_scan_bwd(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"],
                                     x["B"], x["C"], x["dy"], D=x["D"], z=x["z"],
                                     delta_bias=x["delta_bias"], **kw)
    assert scan.mamba_scan_stream_status() == 0
    return g


def oracle_fwd(x):
    return oracle.s6_conv_forward(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"], x["B"],
                                  x["C"], x["delta_bias"], x["D"], x["z"])


def oracle_bwd(x):
    return oracle.s6_conv_backward(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"], x["B"],
                                   x["C"], x["dy"], x["delta_bias"], x["D"], x["z"])


def fwd_case(xh, **kw):
    y, last = gpu_fwd(gc.to_device(xh), **kw)
    y_ref, last_ref = oracle_fwd(xh)
    tol = gc.TOL[xh["u"].dtype]
    ey = gc.normwise(y.cpu().double().numpy(), y_ref)
    el = gc.normwise(last.cpu().double().numpy(), last_ref)
    assert ey <= tol and el <= max(tol, 1e-4), f"y err {ey:.2e}, last_state err {el:.2e}"


def bwd_case(xh, **kw):
    g = gpu_bwd(gc.to_device(xh), **kw)
    ref = oracle_bwd(xh)
    tol = gc.TOL[xh["u"].dtype]
    errs = {k: gc.normwise(g[k].cpu().double().numpy(), ref[k]) for k in GRADS if k in ref}
    assert set(errs) == {k for k in GRADS if k in g}
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"gradient errors above {tol}: {bad} (all: {errs})"


# (batch, dim, L, N): staged kernels (ragged channel groups, several tiles),
# and shapes that go to the one-thread-per-channel kernels (N <= 2, rows that
# are not 16-byte multiples)
STAGED = [(2, 300, 1056, 16), (1, 130, 512, 8), (3, 40, 96, 4), (1, 96, 256, 12)]
REFERENCE = [(2, 37, 50, 2), (1, 20, 33, 16), (2, 9, 40, 1)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", STAGED + REFERENCE, ids=lambda s: "x".join(map(str, s)))
def test_conv_fwd_grid(shape, dtype):
    b, d, L, N = shape
    fwd_case(conv_case(b, d, L, N, dtype, seed=900 + L + d))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", STAGED + REFERENCE, ids=lambda s: "x".join(map(str, s)))
def test_conv_bwd_grid(shape, dtype):
    b, d, L, N = shape
    bwd_case(conv_case(b, d, L, N, dtype, seed=950 + L + d))


@pytest.mark.parametrize("W", [1, 2, 3])
@pytest.mark.parametrize("has_bias", [True, False])
def test_conv_widths_and_bias(W, has_bias):
    x = conv_case(2, 140, 512, 16, torch.float32, W=W, seed=970 + W, has_bias=has_bias)
    fwd_case(x)
    bwd_case(x)


@pytest.mark.parametrize("path", ["reference", "generic"])
def test_conv_explicit_paths(path):
    x = conv_case(1, 130, 256, 16, torch.float32, seed=980)
    fwd_case(x, path=path)
    bwd_case(x, path=path)


@pytest.mark.parametrize("carry", ["sequential", "three_phase"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_conv_fwd_chunks(carry, dtype):
    """Chunks start mid-sequence: their first steps take x from the previous
    chunk, read from memory."""
    fwd_case(conv_case(1, 130, 1024, 16, dtype, seed=985), chunk_len=192, carry=carry)


@pytest.mark.parametrize("chunk_len", [64, 256])
def test_conv_bwd_chunks(chunk_len):
    bwd_case(conv_case(2, 160, 1024, 16, torch.float32, seed=987), chunk_len=chunk_len)


def test_conv_without_gate_and_skip():
    x = conv_case(2, 96, 320, 16, torch.float32, seed=988, has_z=False, has_D=False)
    x["delta_bias"] = None
    fwd_case(x)
    bwd_case(x)


def test_conv_identity_filter_matches_plain_scan_of_silu():
    """With the filter on the current step only and no bias, the prologue is
    u = SiLU(x): the GPU result equals the plain GPU scan on that u."""
    x = gc.to_device(conv_case(2, 200, 512, 16, torch.float32, seed=989))
    x["conv_w"].zero_()
    x["conv_w"][:, 3] = 1.0
    x["conv_b"] = None
    y, last = gpu_fwd(x)
    u = torch.nn.functional.silu(x["u"])
    y2, last2 = scan.selective_scan_fwd(u, x["delta"], x["A"], x["B"], x["C"], D=x["D"],
                                        z=x["z"], delta_bias=x["delta_bias"],
                                        return_last_state=True)
    assert gc.normwise(y.cpu().numpy(), y2.cpu().numpy()) <= 1e-5
    assert gc.normwise(last.cpu().numpy(), last2.cpu().numpy()) <= 1e-5


def test_conv_bwd_deterministic():
    x = gc.to_device(conv_case(2, 300, 1024, 16, torch.bfloat16, seed=990))
    g1, g2 = gpu_bwd(x), gpu_bwd(x)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_conv_full_size_sampled():
    """The bf16 8 x 5120 x 2048 workload with the prologue: y on sampled
    channels against the oracle; dx, ddelta and dz of the backward on sampled
    channels of one batch row; dconv_w, dconv_b on a few channels (summed over
    the whole batch)."""
    w = WORKLOADS[2]
    xh = make_inputs(w.batch, w.dim, w.L, w.N, w.dtype, seed=1236, with_dy=True)
    xh.update(make_conv_params(w.dim, 4, seed=1236))
    x = gc.to_device(xh)
    y, last = gpu_fwd(x)
    g = gpu_bwd(x)
    tol = gc.TOL[w.dtype]
    yh, gh = y.cpu(), {k: v.cpu() for k, v in g.items()}
    per_d = lambda t, idx: None if t is None else t.index_select(0, idx).contiguous()
    for b, ds in gc.sample_channels(w.batch, w.dim, 12, seed=2).items():
        idx = torch.tensor(ds)
        sub = {k: (None if v is None else v[b:b + 1].index_select(1, idx).contiguous())
               for k, v in xh.items() if k in ("u", "delta", "z", "dy")}
        sub.update(B=xh["B"][b:b + 1].contiguous(), C=xh["C"][b:b + 1].contiguous(),
                   A=per_d(xh["A"], idx), D=per_d(xh["D"], idx),
                   delta_bias=per_d(xh["delta_bias"], idx), conv_w=per_d(xh["conv_w"], idx),
                   conv_b=per_d(xh["conv_b"], idx))
        y_ref, _ = oracle_fwd(sub)
        e = gc.normwise(yh[b].index_select(0, idx).double().numpy(), y_ref[0])
        assert e <= tol, f"y (batch {b}): {e:.2e}"
        ref = oracle_bwd(sub)
        for k in ("dx", "ddelta", "dz"):
            e = gc.normwise(gh[k][b].index_select(0, idx).double().numpy(), ref[k][0])
            assert e <= tol, f"{k} (batch {b}): {e:.2e}"
    ds = [0, 2047, w.dim - 1]
    idx = torch.tensor(ds)
    sub = {k: xh[k].index_select(1, idx).contiguous() for k in ("u", "delta", "z", "dy")}
    sub.update(B=xh["B"], C=xh["C"], A=per_d(xh["A"], idx), D=per_d(xh["D"], idx),
               delta_bias=per_d(xh["delta_bias"], idx), conv_w=per_d(xh["conv_w"], idx),
               conv_b=per_d(xh["conv_b"], idx))
    ref = oracle_bwd(sub)
    for k in ("dconv_w", "dconv_b", "dA"):
        e = gc.normwise(gh[k].index_select(0, idx).double().numpy(), ref[k])
        assert e <= tol, f"{k}: {e:.2e}"


def test_conv_rejects_bad_width_and_aliasing():
    x = gc.to_device(conv_case(1, 8, 64, 4, torch.float32, seed=991))
    y = torch.empty_like(x["u"])
    w5 = torch.zeros(8, 5, device="cuda")
    with pytest.raises(scan.MambaScanError) as e:
        scan.mamba_conv_scan_fwd(x["u"], w5, None, x["delta"], x["delta_bias"], x["A"], x["B"],
                                 x["C"], x["D"], x["z"], y, None)
    assert e.value.status == 2  # MAMBA_ERR_UNSUPPORTED
    with pytest.raises(scan.MambaScanError) as e:  # output over an input
        scan.mamba_conv_scan_fwd(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["delta_bias"],
                                 x["A"], x["B"], x["C"], x["D"], x["z"], x["u"], None)
    assert e.value.status == 1  # MAMBA_ERR_INVALID_ARG


@pytest.mark.parametrize("L", [1, 2, 3, 5])
def test_conv_sequences_shorter_than_the_filter(L):
    """L below the filter width: every step sees the zero padding before the
    start (one-thread-per-channel kernels; rows are not 16-byte multiples)."""
    x = conv_case(2, 40, L, 4, torch.float32, seed=992 + L)
    fwd_case(x)
    bwd_case(x)


def test_conv_empty_sequence():
    x = gc.to_device(conv_case(2, 8, 1, 4, torch.float32, seed=996))
    e = {k: (v[..., :0].contiguous() if k in ("u", "delta", "z", "B", "C", "dy") else v)
         for k, v in x.items()}
    y, last = gpu_fwd(e)
    assert y.numel() == 0 and torch.count_nonzero(last) == 0
    g = gpu_bwd(e)
    for k in ("dconv_w", "dconv_b", "dA", "dD", "ddelta_bias"):
        assert torch.count_nonzero(g[k]) == 0, k
