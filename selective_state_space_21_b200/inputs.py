"""Seeded synthetic inputs for the selective scan (S6), shared by both sides.

This module draws random numbers and nothing else: it holds none of the
scan's arithmetic, so that the CUDA path and the fp64 oracle can both be fed
the same values without sharing any computation.

Workloads follow the shapes the Mamba pages describe: d_inner = 2 * d_model
with E = 2 ("Mamba: Linear-Time Sequence Modeling with Selective State
Spaces", paper-graph-ui summary, section 3.4 "The Mamba Architecture"), state
size N = 16 (same page, section 3.6 "State dimension N") and sequences up to
2^20 tokens (Knowl 5 of the chapterpal.com page).  Distributions:

* u, delta, z, B, C, D, dy ~ N(0, 1), drawn as float32 in that order
  (u, delta, z, B, C, D, dt, dy), then cast to the I/O dtype;
* dt per channel log-uniform in [1e-3, 1e-1], and the delta bias set to the
  inverse softplus of dt (the initialisation in section 3.6 "Initialization of
  Delta's bias" of the paper-graph-ui page, with a log-uniform draw);
* A[d, n] = -(n + 1), the S4D-Real initialisation (section 3.6
  "Initialization of A" of the same page), float32.

A, D and the delta bias are always float32; u, delta, z, B, C and dy use the
workload's I/O dtype.

For the convolution prologue of the Mamba block (a short causal convolution
of width d_conv = 4 in front of the S6 layer, Knowl 3 "Mamba Block
Architecture" of the chapterpal.com page) the input x takes the place of u
and is drawn the same way; the per-channel filter and bias are drawn
uniform in [-1/sqrt(W), 1/sqrt(W)] (the usual default initialisation of a
depthwise Conv1d layer, fan-in W; the pages give none).

For the low-rank Delta projection (section 3.6 of the paper-graph-ui page,
s_Delta = Linear_D(Linear_R(x))) the rank-R input dt_low is N(0, 1) and the
weight W_dt is N(0, 1/R), so that their product has delta's unit variance.

For the complex-valued diagonal A (S4D-Lin, A_n = -1/2 + n i, Table 8 of the
paper-graph-ui page's ablations) B and C are complex with N(0, 1/2) real and
imaginary parts, stored planar (real parts first).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int
    L: int
    N: int
    dtype: torch.dtype
    has_z: bool = True
    has_D: bool = True
    backward: bool = False
    description: str = ""

    @property
    def token_channels(self) -> int:
        return self.batch * self.dim * self.L

    @property
    def io_bytes(self) -> int:
        return torch.empty((), dtype=self.dtype).element_size()


#: The five workloads (index = seed offset).  0 is the tiny parity case; 2 is
#: the bf16 2K-length workload that the throughput target is quoted on.
WORKLOADS = [
    Workload("tiny_fp32_b1_d4_L64_N4", 1, 4, 64, 4, torch.float32, backward=True,
             description="tiny fp32 fwd+bwd"),
    Workload("fwd_fp32_b8_d1536_L2048_N16", 8, 1536, 2048, 16, torch.float32,
             description="fp32 fwd at the width of a 768-dim model"),
    Workload("fwd_bf16_b8_d5120_L2048_N16", 8, 5120, 2048, 16, torch.bfloat16,
             description="bf16-I/O fwd at the width of a 2560-dim model"),
    Workload("fwd_bf16_b1_d1536_L1048576_N16", 1, 1536, 1 << 20, 16, torch.bfloat16,
             description="long-sequence bf16 fwd with last_state"),
    Workload("fwdbwd_bf16_b4_d2048_L4096_N16", 4, 2048, 4096, 16, torch.bfloat16,
             backward=True, description="bf16 fwd + recompute bwd"),
]

SEED_BASE = 1234


def inverse_softplus(dt: torch.Tensor) -> torch.Tensor:
    """Value b with log(1 + e^b) = dt, in the stable form dt + log(-expm1(-dt))."""
    return dt + torch.log(-torch.expm1(-dt))


def make_inputs(batch: int, dim: int, L: int, N: int, dtype: torch.dtype = torch.float32,
                device="cpu", seed: int = SEED_BASE, has_z: bool = True, has_D: bool = True,
                with_dy: bool = False, dt_min: float = 1e-3, dt_max: float = 1e-1) -> dict:
    """Draw one set of inputs.  Returns a dict of tensors on ``device``:
    u, delta, z (or None), B, C, A, D (or None), delta_bias and dy (if asked)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    f32 = torch.float32

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=f32)

    u = randn(batch, dim, L).to(dtype)
    delta = randn(batch, dim, L).to(dtype)
    z = randn(batch, dim, L).to(dtype)
    B = randn(batch, N, L).to(dtype)
    C = randn(batch, N, L).to(dtype)
    D = randn(dim)
    r = torch.rand(dim, generator=g, device=device, dtype=f32)
    dt = torch.exp(r * (math.log(dt_max) - math.log(dt_min)) + math.log(dt_min))
    delta_bias = inverse_softplus(dt.double()).to(f32)
    dy = randn(batch, dim, L).to(dtype) if with_dy else None
    A = -torch.arange(1, N + 1, device=device, dtype=f32).repeat(dim, 1).contiguous()
    return {
        "u": u, "delta": delta, "z": z if has_z else None, "B": B, "C": C, "A": A,
        "D": D if has_D else None, "delta_bias": delta_bias, "dy": dy,
    }


def make_conv_params(dim: int, width: int = 4, device="cpu", seed: int = SEED_BASE,
                     has_bias: bool = True) -> dict:
    """Draw a depthwise convolution filter conv_w (dim, width) and bias conv_b
    (dim,) (or None), float32, uniform in [-1/sqrt(width), 1/sqrt(width)]."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 7919)
    bound = 1.0 / math.sqrt(width)
    w = (torch.rand(dim, width, generator=g, device=device) * 2.0 - 1.0) * bound
    b = (torch.rand(dim, generator=g, device=device) * 2.0 - 1.0) * bound
    return {"conv_w": w.contiguous(), "conv_b": b if has_bias else None}


def make_dtproj_params(batch: int, dim: int, L: int, R: int, dtype: torch.dtype = torch.float32,
                       device="cpu", seed: int = SEED_BASE) -> dict:
    """Draw the rank-R input of the low-rank Delta projection, dt_low (batch,
    R, L) ~ N(0, 1), and the weight W_dt (dim, R) ~ N(0, 1/R), both in the I/O
    dtype (so that W_dt . dt_low has unit variance, as delta has)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 104729)
    dt_low = torch.randn(batch, R, L, generator=g, device=device).to(dtype)
    W = (torch.randn(dim, R, generator=g, device=device) / math.sqrt(R)).to(dtype)
    return {"dt_low": dt_low.contiguous(), "W_dt": W.contiguous()}


def make_cplx_inputs(batch: int, dim: int, L: int, N: int, dtype: torch.dtype = torch.float32,
                     device="cpu", seed: int = SEED_BASE, has_z: bool = True, has_D: bool = True,
                     with_dy: bool = False) -> dict:
    """Inputs for the complex-A scan: those of make_inputs (u, delta, z, D,
    delta_bias, dy drawn the same way), with A = S4D-Lin, A[d, n] = -1/2 + n i,
    and B, C complex with N(0, 1/2) real and imaginary parts.  Complex
    vectors are planar, real parts first: A (dim, 2N) float32, B and C (batch,
    2N, L) in the I/O dtype."""
    x = make_inputs(batch, dim, L, N, dtype, device=device, seed=seed, has_z=has_z, has_D=has_D,
                    with_dy=with_dy)
    g = torch.Generator(device=device)
    g.manual_seed(seed + 15485863)
    s = math.sqrt(0.5)
    x["B"] = (torch.randn(batch, 2 * N, L, generator=g, device=device) * s).to(dtype)
    x["C"] = (torch.randn(batch, 2 * N, L, generator=g, device=device) * s).to(dtype)
    n = torch.arange(N, device=device, dtype=torch.float32)
    x["A"] = torch.cat([torch.full((dim, N), -0.5, device=device),
                        n.repeat(dim, 1)], dim=1).contiguous()
    return x


def workload_inputs(index: int, device="cpu", with_dy: Optional[bool] = None) -> dict:
    w = WORKLOADS[index]
    return make_inputs(w.batch, w.dim, w.L, w.N, w.dtype, device=device,
                       seed=SEED_BASE + index, has_z=w.has_z, has_D=w.has_D,
                       with_dy=w.backward if with_dy is None else with_dy)


def gated_case(L: int = 64, dim: int = 4, device="cpu", seed: int = SEED_BASE) -> dict:
    """Theorem-1 case: N = 1, A = -1, B = C = 1, no bias, no D, no z."""
    x = make_inputs(1, dim, L, 1, torch.float32, device=device, seed=seed, has_z=False,
                    has_D=False, with_dy=True)
    x["A"] = -torch.ones(dim, 1, device=device)
    x["B"] = torch.ones(1, 1, L, device=device)
    x["C"] = torch.ones(1, 1, L, device=device)
    x["delta_bias"] = None
    return x


def lti_case(batch: int = 1, dim: int = 4, L: int = 64, N: int = 4, device="cpu",
             seed: int = SEED_BASE, dtype=torch.float32) -> dict:
    """Time-invariant case: delta, B and C held at their t = 0 values."""
    x = make_inputs(batch, dim, L, N, dtype, device=device, seed=seed, with_dy=True)
    for k in ("delta",):
        x[k] = x[k][:, :, :1].expand(batch, dim, L).contiguous()
    for k in ("B", "C"):
        x[k] = x[k][:, :, :1].expand(batch, N, L).contiguous()
    return x
