"""GPU parity of the decoding step (mamba_scan_step, one token per call)
against the fp64 oracle: stepping token by token reproduces the full-sequence
scan, continuing from a forward's last_state (prefill, then decode) does too,
and one step from an arbitrary state matches the oracle started from it."""
import numpy as np
import pytest
import torch

import gpu_cases as gc
import oracle
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import make_conv_params, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()


def _token(x, t):
    pick = lambda k: None if x[k] is None else x[k][:, :, t].contiguous()
    return {k: pick(k) for k in ("u", "delta", "z", "B", "C")}


def _decode(x, state, t0, t1):
    ys = []
    for t in range(t0, t1):
        tok = _token(x, t)
        y = torch.empty_like(tok["u"])
        scan.mamba_scan_step(state, tok["u"], tok["delta"], x["delta_bias"], x["A"], tok["B"],
                             tok["C"], x["D"], tok["z"], y)
        ys.append(y)
    assert scan.mamba_scan_stream_status() == 0
    return torch.stack(ys, dim=-1)


SHAPES = [(2, 200, 24, 16), (1, 37, 10, 3), (3, 20, 9, 8), (1, 5, 12, 1)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_decode_token_by_token_matches_full_scan(shape, dtype):
    b, d, L, N = shape
    xh = make_inputs(b, d, L, N, dtype, seed=800 + L + d)
    x = gc.to_device(xh)
    state = torch.zeros(b, d, N, device="cuda")
    y = _decode(x, state, 0, L)
    y_ref, last_ref = gc.oracle_fwd(xh)
    tol = gc.TOL[dtype]
    assert gc.normwise(y.cpu().double().numpy(), y_ref) <= tol
    assert gc.normwise(state.cpu().double().numpy(), last_ref) <= max(tol, 1e-4)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_prefill_with_forward_then_decode(dtype):
    """The forward over a prompt leaves last_state; decoding continues from it."""
    b, d, L, N, L1 = 2, 300, 1056, 16, 1024
    xh = make_inputs(b, d, L, N, dtype, seed=901)
    x = gc.to_device(xh)
    prompt = {k: (v[..., :L1].contiguous() if k in ("u", "delta", "z", "B", "C") and v is not None
                  else v) for k, v in x.items()}
    y1, state = gc.gpu_fwd(prompt)
    y2 = _decode(x, state, L1, L)
    y_ref, last_ref = gc.oracle_fwd(xh)
    tol = gc.TOL[dtype]
    y = torch.cat([y1, y2], dim=-1)
    assert gc.normwise(y.cpu().double().numpy(), y_ref) <= tol
    assert gc.normwise(y2.cpu().double().numpy(), y_ref[..., L1:]) <= tol
    assert gc.normwise(state.cpu().double().numpy(), last_ref) <= max(tol, 1e-4)


def test_one_step_from_an_arbitrary_state():
    b, d, N = 4, 130, 16
    xh = make_inputs(b, d, 1, N, torch.float32, seed=902)
    h0 = torch.randn(b, d, N, generator=torch.Generator().manual_seed(5))
    x = gc.to_device(xh)
    state = h0.cuda()
    y = _decode(x, state, 0, 1)
    y_ref, last_ref = oracle.s6_forward(xh["u"], xh["delta"], xh["A"], xh["B"], xh["C"],
                                        xh["delta_bias"], xh["D"], xh["z"], initial_state=h0)
    assert gc.normwise(y.cpu().double().numpy(), y_ref) <= 1e-4
    assert gc.normwise(state.cpu().double().numpy(), last_ref) <= 1e-4


def test_step_rejects_overlapping_state_and_output():
    b, d, N = 1, 8, 4
    x = gc.to_device(make_inputs(b, d, 1, N, torch.float32, seed=3))
    tok = _token(x, 0)
    state = torch.zeros(b * d * N + b * d, device="cuda")
    st, y = state[: b * d * N].view(b, d, N), state[b * d * N - 2: b * d * N - 2 + b * d].view(b, d)
    with pytest.raises(scan.MambaScanError) as e:
        scan.mamba_scan_step(st, tok["u"], tok["delta"], x["delta_bias"], x["A"], tok["B"],
                             tok["C"], x["D"], tok["z"], y)
    assert e.value.status == 1


def _conv_decode(x, state, conv_state, t0, t1):
    ys = []
    for t in range(t0, t1):
        tok = _token(x, t)
        y = torch.empty_like(tok["u"])
        scan.mamba_conv_scan_step(state, conv_state, tok["u"], x["conv_w"], x["conv_b"],
                                  tok["delta"], x["delta_bias"], x["A"], tok["B"], tok["C"],
                                  x["D"], tok["z"], y)
        ys.append(y)
    assert scan.mamba_scan_stream_status() == 0
    return torch.stack(ys, dim=-1)


def _conv_oracle(xh):
    return oracle.s6_conv_forward(xh["u"], xh["conv_w"], xh["conv_b"], xh["delta"], xh["A"],
                                  xh["B"], xh["C"], xh["delta_bias"], xh["D"], xh["z"])


@pytest.mark.parametrize("W", [4, 3, 2, 1])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 200, 24, 16), (1, 37, 10, 3)],
                         ids=lambda s: "x".join(map(str, s)))
def test_conv_decode_token_by_token_matches_full_conv_scan(shape, dtype, W):
    """Stepping the block with its convolution state from zeros reproduces
    the full-sequence forward with the prologue."""
    b, d, L, N = shape
    xh = make_inputs(b, d, L, N, dtype, seed=860 + L + W)
    xh.update(make_conv_params(d, W, seed=860 + W))
    x = gc.to_device(xh)
    state = torch.zeros(b, d, N, device="cuda")
    conv_state = torch.zeros(b, d, W - 1, device="cuda")
    y = _conv_decode(x, state, conv_state, 0, L)
    y_ref, last_ref = _conv_oracle(xh)
    tol = gc.TOL[dtype]
    assert gc.normwise(y.cpu().double().numpy(), y_ref) <= tol
    assert gc.normwise(state.cpu().double().numpy(), last_ref) <= max(tol, 1e-4)
    if W > 1:  # the state holds the last W - 1 inputs
        assert torch.equal(conv_state.cpu(), xh["u"][..., L - W + 1:].float())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_conv_prefill_then_decode(dtype):
    """The fused forward over a prompt leaves last_state; with the prompt's
    last three inputs as the convolution state, decoding continues it."""
    b, d, L, N, L1 = 2, 300, 1056, 16, 1024
    xh = make_inputs(b, d, L, N, dtype, seed=902)
    xh.update(make_conv_params(d, 4, seed=902))
    x = gc.to_device(xh)
    prompt = {k: (v[..., :L1].contiguous() if k in ("u", "delta", "z", "B", "C") and v is not None
                  else v) for k, v in x.items()}
    y1, state = scan.conv_selective_scan_fwd(prompt["u"], x["conv_w"], x["conv_b"],
                                             prompt["delta"], x["A"], prompt["B"], prompt["C"],
                                             D=x["D"], z=prompt["z"], delta_bias=x["delta_bias"],
                                             return_last_state=True)
    conv_state = x["u"][..., L1 - 3:L1].float().contiguous()
    y2 = _conv_decode(x, state, conv_state, L1, L)
    y_ref, last_ref = _conv_oracle(xh)
    tol = gc.TOL[dtype]
    assert gc.normwise(torch.cat([y1, y2], dim=-1).cpu().double().numpy(), y_ref) <= tol
    assert gc.normwise(y2.cpu().double().numpy(), y_ref[..., L1:]) <= tol
    assert gc.normwise(state.cpu().double().numpy(), last_ref) <= max(tol, 1e-4)
