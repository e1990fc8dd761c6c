"""Independent checks that pin the fp64 oracle to what the pages and the
mathematics fix.  None of these re-types the oracle's loop: each one computes
the same quantity a different way (a closed form, a library routine, an
unrolled sum, the continuous-time solution, finite differences or autograd).

Every function returns ``(error, tolerance)``; ``run_all(lib)`` runs them all
against a given oracle library (the real one, or a deliberately broken copy in
the mutation test).
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import scipy.linalg
import scipy.signal
import scipy.special
import torch

import oracle
from selective_state_space_21_b200.inputs import (gated_case, lti_case, make_conv_params,
                                                  make_cplx_inputs, make_inputs)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_derived_exact.txt")


def _np(x):
    return None if x is None else x.detach().cpu().double().numpy()


def normwise(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = max(np.abs(ref).max(initial=0.0), 1e-300)
    return float(np.abs(got - ref).max(initial=0.0) / scale)


def _softplus(v):
    return np.logaddexp(0.0, v)  # numpy's own log(e^0 + e^v)


# ------------------------------------------------------------------ golden

def _parse_value(tok: str) -> float:
    neg = tok.startswith("-")
    body = tok[1:] if neg else tok
    if body.startswith("ln"):
        v = math.log(float(body[2:]))
    else:
        v = float(Fraction(body))
    return -v if neg else v


def load_golden():
    cases, cur = [], None
    with open(GOLDEN) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "case":
                cur = {"name": vals[0]}
                cases.append(cur)
            else:
                cur[key] = [_parse_value(v) for v in vals]
    return cases


def pin_golden(lib=None):
    """Hand-derived exact values (Theorem 1 and held-input zero-order hold)."""
    worst = 0.0
    for c in load_golden():
        N = int(c["N"][0])
        L = len(c["u"])
        u = np.array(c["u"]).reshape(1, 1, L)
        delta = np.array(c["delta"]).reshape(1, 1, L)
        A = np.array(c["A"]).reshape(1, N)
        B = np.repeat(np.array(c["B"]).reshape(1, N, 1), L, axis=2)
        C = np.repeat(np.array(c["C"]).reshape(1, N, 1), L, axis=2)
        bias = np.array(c["delta_bias"])
        y, _ = oracle.s6_forward(u, delta, A, B, C, delta_bias=bias, lib=lib, nthreads=1)
        worst = max(worst, normwise(y.ravel(), np.array(c["y"])))
    return worst, 1e-14


# ------------------------------------------------------------- Theorem 1

def pin_theorem1(lib=None):
    """N=1, A=-1, B=C=1, no bias: h_t = (1-g_t) h_{t-1} + g_t u_t, g = sigma(delta)."""
    x = gated_case(L=257, dim=3)
    y, last = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], lib=lib)
    u, d = _np(x["u"]), _np(x["delta"])
    g = scipy.special.expit(d)
    h = np.zeros(u.shape[:2])
    ref = np.empty_like(u)
    for t in range(u.shape[2]):
        h = (1.0 - g[..., t]) * h + g[..., t] * u[..., t]
        ref[..., t] = h
    return max(normwise(y, ref), normwise(last[..., 0], h)), 1e-13


# ------------------------------------------- ZOH by the matrix exponential

def _zoh_expm(Delta, Avec, Bvec):
    """Zero-order hold of h' = diag(A) h + B x over a step Delta via the
    augmented-matrix exponential (Van Loan), with no diagonal shortcut."""
    N = Avec.shape[0]
    M = np.zeros((N + 1, N + 1))
    M[:N, :N] = np.diag(Avec) * Delta
    M[:N, N] = Bvec * Delta
    E = scipy.linalg.expm(M)
    return E[:N, :N], E[:N, N]


def pin_zoh_expm(lib=None):
    """Time-varying Delta, B, C; discretized step by step with scipy's expm."""
    x = make_inputs(2, 3, 40, 4, seed=77, with_dy=False)
    x["A"] = -torch.rand(3, 4, generator=torch.Generator().manual_seed(5)) * 3.0 - 0.05
    y, last = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                x["D"], x["z"], lib=lib)
    u, dl, z = _np(x["u"]), _np(x["delta"]), _np(x["z"])
    A, B, C, D, bias = _np(x["A"]), _np(x["B"]), _np(x["C"]), _np(x["D"]), _np(x["delta_bias"])
    ref = np.empty_like(u)
    ref_last = np.empty(last.shape)
    for b in range(u.shape[0]):
        for d in range(u.shape[1]):
            h = np.zeros(A.shape[1])
            for t in range(u.shape[2]):
                Abar, Bbar = _zoh_expm(_softplus(dl[b, d, t] + bias[d]), A[d], B[b, :, t])
                h = Abar @ h + Bbar * u[b, d, t]
                y0 = C[b, :, t] @ h + D[d] * u[b, d, t]
                ref[b, d, t] = y0 * z[b, d, t] * scipy.special.expit(z[b, d, t])
            ref_last[b, d] = h
    return max(normwise(y, ref), normwise(last, ref_last)), 1e-12


# ---------------------------------------------- LTI <=> global convolution

def pin_lti_convolution(lib=None):
    """Constant Delta, B, C: y0 = (x * K) + D x with K_k = C Abar^k Bbar, the
    discretization taken from scipy.signal.cont2discrete(method='zoh')."""
    x = lti_case(batch=2, dim=3, L=96, N=5, seed=91)
    y, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                             x["D"], x["z"], lib=lib)
    u, dl, z = _np(x["u"]), _np(x["delta"]), _np(x["z"])
    A, B, C, D, bias = _np(x["A"]), _np(x["B"]), _np(x["C"]), _np(x["D"]), _np(x["delta_bias"])
    L = u.shape[2]
    ref = np.empty_like(u)
    for b in range(u.shape[0]):
        for d in range(u.shape[1]):
            Delta = float(_softplus(dl[b, d, 0] + bias[d]))
            sysd = scipy.signal.cont2discrete(
                (np.diag(A[d]), B[b, :, 0:1], C[b, :, 0:1].T, np.zeros((1, 1))), Delta,
                method="zoh")
            Ad, Bd = sysd[0], sysd[1][:, 0]
            K = np.empty(L)
            p = Bd.copy()
            for k in range(L):
                K[k] = C[b, :, 0] @ p
                p = Ad @ p
            y0 = np.convolve(u[b, d], K)[:L] + D[d] * u[b, d]
            ref[b, d] = y0 * z[b, d] * scipy.special.expit(z[b, d])
    return normwise(y, ref), 1e-12


# ----------------------------------------------------- brute-force unroll

def pin_brute_force(lib=None):
    """y0_t = sum_{k<=t} sum_n C_tn exp(A_n (S_t - S_k)) Bbar_kn u_k + D u_t,
    S the running sum of Delta (the product of Abar over (k, t] in closed form)."""
    x = make_inputs(1, 4, 64, 4, seed=4242, with_dy=False)
    y, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                             x["D"], x["z"], lib=lib)
    u, dl, z = _np(x["u"]), _np(x["delta"]), _np(x["z"])
    A, B, C, D, bias = _np(x["A"]), _np(x["B"]), _np(x["C"]), _np(x["D"]), _np(x["delta_bias"])
    L = u.shape[2]
    ref = np.empty_like(u)
    for d in range(u.shape[1]):
        Delta = _softplus(dl[0, d] + bias[d])
        S = np.cumsum(Delta)
        for t in range(L):
            acc = D[d] * u[0, d, t]
            for k in range(t + 1):
                for n in range(A.shape[1]):
                    a = A[d, n]
                    bbar = (math.exp(Delta[k] * a) - 1.0) / a * B[0, n, k]
                    acc += C[0, n, t] * math.exp(a * (S[t] - S[k])) * bbar * u[0, d, k]
            ref[0, d, t] = acc * z[0, d, t] * scipy.special.expit(z[0, d, t])
    return normwise(y, ref), 1e-11


# ------------------------------------------- held input: exact ODE solution

def pin_held_input_exact(lib=None):
    """u = 1, B = 1, C = 1, time-varying Delta: zero-order hold is exact for a
    held input, so h_n(t) = (exp(A_n T_t) - 1) / A_n with T_t = sum_{j<=t} Delta_j."""
    x = make_inputs(1, 3, 200, 6, seed=303, has_z=False, has_D=False)
    L, N = 200, 6
    A = -(np.arange(1, N + 1)[None, :] * np.array([[0.5], [1.0], [2.0]]))
    u = np.ones((1, 3, L))
    ones = np.ones((1, N, L))
    y, last = oracle.s6_forward(u, x["delta"], A, ones, ones, x["delta_bias"], lib=lib)
    Delta = _softplus(_np(x["delta"])[0] + _np(x["delta_bias"])[:, None])
    T = np.cumsum(Delta, axis=1)  # (dim, L)
    ref = np.sum((np.exp(A[:, :, None] * T[:, None, :]) - 1.0) / A[:, :, None], axis=1)
    return normwise(y[0], ref), 1e-12


# ------------------------------------------------------ skip, gate, limits

def pin_skip_and_gate(lib=None):
    """C = 0 leaves y = D u silu(z) exactly; silu(z) = z sigma(z) (SiLU as the
    pages define it), with sigma from scipy.special.expit."""
    x = make_inputs(2, 5, 33, 3, seed=11)
    zeros = torch.zeros_like(x["C"])
    y, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], zeros, x["delta_bias"],
                             x["D"], x["z"], lib=lib)
    u, z, D = _np(x["u"]), _np(x["z"]), _np(x["D"])
    ref = D[None, :, None] * u * z * scipy.special.expit(z)
    e1 = normwise(y, ref)
    # the gate multiplies the ungated output
    y_gated, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                   x["D"], x["z"], lib=lib)
    y_plain, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                   x["D"], None, lib=lib)
    e2 = normwise(y_gated, y_plain * z * scipy.special.expit(z))
    return max(e1, e2), 1e-14


def pin_large_delta_limit(lib=None):
    """Large Delta resets the state (Knowl 4 mechanics): h_t -> -B_t u_t / A."""
    x = make_inputs(1, 3, 50, 4, seed=12, has_z=False)
    bias = torch.full((3,), 60.0)
    y, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], bias, x["D"], lib=lib)
    u, B, C, A, D = _np(x["u"]), _np(x["B"]), _np(x["C"]), _np(x["A"]), _np(x["D"])
    h = -B[:, None, :, :] * u[:, :, None, :] / A[None, :, :, None]
    ref = np.einsum("bnt,bdnt->bdt", C, h) + D[None, :, None] * u
    return normwise(y, ref), 1e-12


def pin_small_delta_limit(lib=None):
    """Small Delta keeps the state and lets the input in at rate Delta:
    h_t ~= sum_{k<=t} Delta_k B_k u_k, to first order in Delta."""
    x = make_inputs(1, 3, 50, 4, seed=13, has_z=False, has_D=False)
    bias = torch.full((3,), -30.0)  # Delta ~ 1e-13
    y, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], bias, lib=lib)
    u, dl, B, C = _np(x["u"]), _np(x["delta"]), _np(x["B"]), _np(x["C"])
    Delta = _softplus(dl + _np(bias)[None, :, None])
    h = np.cumsum(Delta[:, :, None, :] * B[:, None, :, :] * u[:, :, None, :], axis=3)
    ref = np.einsum("bnt,bdnt->bdt", C, h)
    return normwise(y, ref), 1e-10


def pin_structure(lib=None):
    """Causality, linearity in u and independence of channels and batches."""
    x = make_inputs(2, 4, 48, 4, seed=21)
    args = lambda u: (u, x["delta"], x["A"], x["B"], x["C"], x["delta_bias"], x["D"], x["z"])
    y, _ = oracle.s6_forward(*args(x["u"]), lib=lib)
    errs = []
    # causality: perturbing u at t0 leaves y_{<t0} untouched
    u2 = x["u"].clone()
    u2[:, :, 30] += 1.0
    y2, _ = oracle.s6_forward(*args(u2), lib=lib)
    errs.append(float(np.abs(y2[:, :, :30] - y[:, :, :30]).max()))
    errs.append(0.0 if np.abs(y2[:, :, 30:] - y[:, :, 30:]).max() > 1e-6 else 1.0)
    # linearity in u (z, delta, B, C fixed)
    ua = torch.randn(x["u"].shape, generator=torch.Generator().manual_seed(3), dtype=torch.float64)
    ub = torch.randn(x["u"].shape, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
    ya, _ = oracle.s6_forward(*args(ua), lib=lib)
    yb, _ = oracle.s6_forward(*args(ub), lib=lib)
    yab, _ = oracle.s6_forward(*args(2.0 * ua - 3.0 * ub), lib=lib)
    errs.append(normwise(yab, 2.0 * ya - 3.0 * yb))
    # channel and batch independence
    u3 = x["u"].clone()
    u3[1, 2] += 5.0
    y3, _ = oracle.s6_forward(*args(u3), lib=lib)
    mask = np.ones(y.shape, bool)
    mask[1, 2] = False
    errs.append(float(np.abs(y3 - y)[mask].max()))
    return max(errs), 1e-12


# -------------------------------------------------------------- backward

def _fd_inputs():
    x = make_inputs(1, 2, 10, 3, seed=31, with_dy=True)
    x = {k: (v.double() if v is not None else None) for k, v in x.items()}
    x["A"] = x["A"] * 0.7  # a generic (non-integer) diagonal
    return x


def _loss(x, lib):
    y, _ = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                             x["D"], x["z"], lib=lib, nthreads=1)
    return float(np.sum(_np(x["dy"]) * y))


_GRAD_NAMES = {"u": "du", "delta": "ddelta", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
               "D": "dD", "delta_bias": "ddelta_bias"}


def pin_finite_differences(lib=None):
    """Central differences of sum(dy * y) over every scalar input."""
    x = _fd_inputs()
    g = oracle.s6_backward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"],
                           x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    worst = 0.0
    for name, gname in _GRAD_NAMES.items():
        base = x[name]
        fd = np.empty(base.shape)
        flat = base.reshape(-1)
        for i in range(flat.numel()):
            v = float(flat[i])
            h = 1e-6 * max(1.0, abs(v))
            flat[i] = v + h
            lp = _loss(x, lib)
            flat[i] = v - h
            lm = _loss(x, lib)
            flat[i] = v
            fd.reshape(-1)[i] = (lp - lm) / (2.0 * h)
        worst = max(worst, normwise(g[gname], fd))
    return worst, 1e-6


def _torch_forward(x):
    """A plain float64 torch forward used only so that autograd can supply
    gradients by its own rules (it checks the hand-derived adjoint)."""
    u, dl, z = x["u"], x["delta"], x["z"]
    A, B, C, D, bias = x["A"], x["B"], x["C"], x["D"], x["delta_bias"]
    Delta = torch.nn.functional.softplus(dl + bias[None, :, None], beta=1.0, threshold=1e9)
    h = torch.zeros(u.shape[0], u.shape[1], A.shape[1], dtype=torch.float64)
    ys = []
    for t in range(u.shape[2]):
        dA = Delta[:, :, t, None] * A[None]
        Abar = torch.matrix_exp(torch.diag_embed(dA)).diagonal(dim1=-2, dim2=-1)
        Bbar = (Abar - 1.0) / A[None] * B[:, None, :, t]
        h = Abar * h + Bbar * u[:, :, t, None]
        y0 = (h * C[:, None, :, t]).sum(-1) + D[None] * u[:, :, t]
        ys.append(y0 * torch.nn.functional.silu(z[:, :, t]))
    return torch.stack(ys, dim=-1)


def pin_autograd(lib=None):
    """The adjoint against torch.autograd of an independent float64 forward."""
    x = _fd_inputs()
    leaves = {k: x[k].clone().requires_grad_(True) for k in _GRAD_NAMES}
    y = _torch_forward({**x, **leaves})
    (y * x["dy"]).sum().backward()
    g = oracle.s6_backward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"],
                           x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    worst = 0.0
    for name, gname in _GRAD_NAMES.items():
        worst = max(worst, normwise(g[gname], leaves[name].grad.numpy()))
    return worst, 1e-10


def pin_threads_agree(lib=None):
    """The multithreaded oracle gives the single-threaded result bit for bit."""
    x = make_inputs(3, 7, 40, 4, seed=8, with_dy=True)
    a = (x["u"], x["delta"], x["A"], x["B"], x["C"])
    kw = dict(delta_bias=x["delta_bias"], D=x["D"], z=x["z"], lib=lib)
    y1, l1 = oracle.s6_forward(*a, nthreads=1, **kw)
    y4, l4 = oracle.s6_forward(*a, nthreads=4, **kw)
    g1 = oracle.s6_backward(*a, x["dy"], nthreads=1, **kw)
    g4 = oracle.s6_backward(*a, x["dy"], nthreads=4, **kw)
    err = max(float(np.abs(y1 - y4).max()), float(np.abs(l1 - l4).max()))
    for k in ("du", "ddelta", "dz", "dA", "dD", "ddelta_bias"):
        err = max(err, float(np.abs(g1[k] - g4[k]).max()))
    for k in ("dB", "dC"):  # summed over channels in a different grouping
        err = max(err, normwise(g4[k], g1[k]) * 1e-3)
    return err, 1e-15


def pin_resume_from_state(lib=None):
    """Splitting a sequence and continuing from the first part's final state
    gives the unsplit result (the recurrence carries everything in h)."""
    x = make_inputs(2, 3, 50, 4, seed=61)
    sl = lambda t, a, b: None if t is None else t[..., a:b].contiguous()
    full, last = oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                   x["D"], x["z"], lib=lib)
    args = lambda a, b: (sl(x["u"], a, b), sl(x["delta"], a, b), x["A"], sl(x["B"], a, b),
                         sl(x["C"], a, b), x["delta_bias"], x["D"], sl(x["z"], a, b))
    y1, h1 = oracle.s6_forward(*args(0, 21), lib=lib)
    y2, h2 = oracle.s6_forward(*args(21, 50), lib=lib, initial_state=h1)
    e = max(normwise(np.concatenate([y1, y2], axis=2), full), normwise(h2, last))
    return e, 1e-14


def pin_initial_state_decay(lib=None):
    """With u = 0 a starting state only decays: h_L = exp(A sum_t Delta_t) h_0."""
    x = make_inputs(1, 3, 30, 5, seed=62, has_z=False, has_D=False)
    h0 = np.random.default_rng(7).standard_normal((1, 3, 5))
    zeros = torch.zeros_like(x["u"])
    _, last = oracle.s6_forward(zeros, x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                lib=lib, initial_state=h0)
    Delta = _softplus(_np(x["delta"])[0] + _np(x["delta_bias"])[:, None])
    ref = np.exp(_np(x["A"]) * Delta.sum(axis=1)[:, None]) * h0[0]
    return normwise(last[0], ref), 1e-13


# ------------------------------------------------- convolution prologue

def _silu(p):
    return p * scipy.special.expit(p)  # scipy's logistic function


def pin_conv_numpy(lib=None):
    """The causal depthwise convolution against numpy's full convolution
    (flipped filter, first L outputs) and SiLU through scipy's logistic."""
    worst = 0.0
    for W, seed, has_bias in ((4, 71, True), (3, 72, False), (1, 73, True), (2, 74, True)):
        x = make_inputs(2, 3, 37, 2, seed=seed)["u"].double().numpy()
        cp = make_conv_params(3, W, seed=seed, has_bias=has_bias)
        w = cp["conv_w"].double().numpy()
        cb = None if cp["conv_b"] is None else cp["conv_b"].double().numpy()
        pre, u = oracle.conv_silu(x, w, cb, lib=lib)
        ref = np.empty_like(x)
        for b in range(2):
            for d in range(3):
                ref[b, d] = np.convolve(x[b, d], w[d, ::-1])[:37] + (cb[d] if cb is not None else 0.0)
        worst = max(worst, normwise(pre, ref), normwise(u, _silu(ref)))
    return worst, 1e-14


def pin_conv_special_filters(lib=None):
    """An identity filter (weight only on the current step, no bias) makes
    the prologue u = SiLU(x); a filter on the oldest step makes it
    u_t = SiLU(x_{t-3}) with zeros before the start.  Both then equal the
    plain forward on that u."""
    xi = make_inputs(2, 3, 29, 4, seed=75)
    x = xi["u"].double().numpy()
    common = dict(delta_bias=xi["delta_bias"], D=xi["D"], z=xi["z"], lib=lib)
    worst = 0.0
    for k_on, shift in ((3, 0), (0, 3)):
        w = np.zeros((3, 4))
        w[:, k_on] = 1.0
        y, last = oracle.s6_conv_forward(x, w, None, xi["delta"], xi["A"], xi["B"], xi["C"],
                                         **common)
        u = np.zeros_like(x)
        u[..., shift:] = _silu(x[..., :x.shape[2] - shift])
        y_ref, last_ref = oracle.s6_forward(u, xi["delta"], xi["A"], xi["B"], xi["C"], **common)
        worst = max(worst, normwise(y, y_ref), normwise(last, last_ref))
    return worst, 1e-14


def _conv_fd_inputs():
    x = make_inputs(1, 2, 10, 3, seed=76, with_dy=True)
    x = {k: (v.double() if v is not None else None) for k, v in x.items()}
    x["A"] = x["A"] * 0.7
    cp = make_conv_params(2, 4, seed=76)
    x["conv_w"] = cp["conv_w"].double()
    x["conv_b"] = cp["conv_b"].double()
    return x


def _conv_loss(x, lib):
    y, _ = oracle.s6_conv_forward(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"], x["B"],
                                  x["C"], x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    return float(np.sum(_np(x["dy"]) * y))


def _conv_grads(x, lib):
    return oracle.s6_conv_backward(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["A"], x["B"],
                                   x["C"], x["dy"], x["delta_bias"], x["D"], x["z"], lib=lib,
                                   nthreads=1)


def pin_conv_finite_differences(lib=None):
    """Central differences of sum(dy * y) through the prologue: x, the filter,
    its bias, and delta and A behind it."""
    x = _conv_fd_inputs()
    g = _conv_grads(x, lib)
    names = {"u": "dx", "conv_w": "dconv_w", "conv_b": "dconv_b", "delta": "ddelta", "A": "dA"}
    worst = 0.0
    for name, gname in names.items():
        flat = x[name].reshape(-1)
        fd = np.empty(x[name].shape)
        for i in range(flat.numel()):
            v = float(flat[i])
            h = 1e-6 * max(1.0, abs(v))
            flat[i] = v + h
            lp = _conv_loss(x, lib)
            flat[i] = v - h
            lm = _conv_loss(x, lib)
            flat[i] = v
            fd.reshape(-1)[i] = (lp - lm) / (2.0 * h)
        worst = max(worst, normwise(g[gname], fd))
    return worst, 1e-6


def pin_conv_autograd(lib=None):
    """The prologue's chain rule against torch.autograd through torch's own
    conv1d (causal by left padding, depthwise by groups) and silu, fed with
    the (separately pinned) S6 gradient du at the prologue's output."""
    x = _conv_fd_inputs()
    xs = x["u"].clone().requires_grad_(True)
    w = x["conv_w"].clone().requires_grad_(True)
    cb = x["conv_b"].clone().requires_grad_(True)
    dim, W = w.shape
    L = xs.shape[2]
    pre = torch.nn.functional.conv1d(xs, w[:, None, :], cb, padding=W - 1, groups=dim)[..., :L]
    u = torch.nn.functional.silu(pre)
    gs6 = oracle.s6_backward(u.detach(), x["delta"], x["A"], x["B"], x["C"], x["dy"],
                             x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    ref = torch.autograd.grad(u, (xs, w, cb), grad_outputs=torch.from_numpy(gs6["du"]))
    g = _conv_grads(x, lib)
    worst = 0.0
    for got, r in zip((g["dx"], g["dconv_w"], g["dconv_b"]), ref):
        worst = max(worst, normwise(got, r.numpy()))
    return worst, 1e-12


# -------------------------------------------- low-rank Delta projection

def _dtproj_inputs(seed, b=2, d=3, L=23, N=4, R=2):
    x = make_inputs(b, d, L, N, seed=seed, with_dy=True)
    x = {k: (v.double() if v is not None else None) for k, v in x.items()}
    g = torch.Generator().manual_seed(seed)
    x["dt_low"] = torch.randn(b, R, L, generator=g, dtype=torch.float64)
    x["W_dt"] = torch.randn(d, R, generator=g, dtype=torch.float64) / math.sqrt(R)
    return x


def pin_dtproj_matmul(lib=None):
    """The projection against numpy's einsum: delta = W_dt . dt_low, then the
    plain forward on that delta."""
    x = _dtproj_inputs(81, R=5)
    y, last = oracle.s6_dtproj_forward(x["u"], x["dt_low"], x["W_dt"], x["A"], x["B"], x["C"],
                                       x["delta_bias"], x["D"], x["z"], lib=lib)
    delta = np.einsum("dr,brl->bdl", _np(x["W_dt"]), _np(x["dt_low"]))
    y_ref, last_ref = oracle.s6_forward(x["u"], delta, x["A"], x["B"], x["C"], x["delta_bias"],
                                        x["D"], x["z"], lib=lib)
    return max(normwise(y, y_ref), normwise(last, last_ref)), 1e-13


def _dtproj_loss(x, lib):
    y, _ = oracle.s6_dtproj_forward(x["u"], x["dt_low"], x["W_dt"], x["A"], x["B"], x["C"],
                                    x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    return float(np.sum(_np(x["dy"]) * y))


def pin_dtproj_finite_differences(lib=None):
    """Central differences of sum(dy * y) through the projection: dt_low,
    W_dt and u."""
    x = _dtproj_inputs(82, b=1, d=2, L=9, N=3, R=2)
    g = oracle.s6_dtproj_backward(x["u"], x["dt_low"], x["W_dt"], x["A"], x["B"], x["C"],
                                  x["dy"], x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    worst = 0.0
    for name, gname in {"dt_low": "d_dt_low", "W_dt": "dW_dt", "u": "du"}.items():
        flat = x[name].reshape(-1)
        fd = np.empty(x[name].shape)
        for i in range(flat.numel()):
            v = float(flat[i])
            h = 1e-6 * max(1.0, abs(v))
            flat[i] = v + h
            lp = _dtproj_loss(x, lib)
            flat[i] = v - h
            lm = _dtproj_loss(x, lib)
            flat[i] = v
            fd.reshape(-1)[i] = (lp - lm) / (2.0 * h)
        worst = max(worst, normwise(g[gname], fd))
    return worst, 1e-6


def pin_dtproj_autograd(lib=None):
    """The projection's chain rule against torch.autograd through torch's
    matmul, fed with the (separately pinned) S6 gradient ddelta."""
    x = _dtproj_inputs(83, R=3)
    dl = x["dt_low"].clone().requires_grad_(True)
    W = x["W_dt"].clone().requires_grad_(True)
    delta = torch.matmul(W, dl)  # (d, R) @ (b, R, L) -> (b, d, L)
    gs6 = oracle.s6_backward(x["u"], delta.detach(), x["A"], x["B"], x["C"], x["dy"],
                             x["delta_bias"], x["D"], x["z"], lib=lib)
    ref = torch.autograd.grad(delta, (dl, W), grad_outputs=torch.from_numpy(gs6["ddelta"]))
    g = oracle.s6_dtproj_backward(x["u"], x["dt_low"], x["W_dt"], x["A"], x["B"], x["C"],
                                  x["dy"], x["delta_bias"], x["D"], x["z"], lib=lib)
    return max(normwise(g["d_dt_low"], ref[0].numpy()), normwise(g["dW_dt"], ref[1].numpy())), 1e-12


# ------------------------------------------------- complex diagonal A

def _cplx(x, N):
    """planar (..., 2N, ...) along axis -2 or -1 -> complex numpy array"""
    return x[..., :N] + 1j * x[..., N:]


def pin_cplx_real_case(lib=None):
    """With zero imaginary parts the complex scan is the real one: y, the
    state and the real-part gradients equal the (separately pinned) real
    oracle's."""
    xr = make_inputs(2, 3, 31, 4, seed=91, with_dy=True)
    xr["A"] = xr["A"] * 0.6
    N = 4
    z2 = lambda t: torch.cat([t, torch.zeros_like(t)], dim=-2)  # (b, N, L) -> (b, 2N, L)
    A2 = torch.cat([xr["A"], torch.zeros_like(xr["A"])], dim=1)
    kw = dict(delta_bias=xr["delta_bias"], D=xr["D"], z=xr["z"], lib=lib)
    y, last = oracle.s6_cplx_forward(xr["u"], xr["delta"], A2, z2(xr["B"]), z2(xr["C"]), **kw)
    y_r, last_r = oracle.s6_forward(xr["u"], xr["delta"], xr["A"], xr["B"], xr["C"], **kw)
    err = max(normwise(y, y_r), normwise(last[..., :N], last_r), float(np.abs(last[..., N:]).max()))
    g = oracle.s6_cplx_backward(xr["u"], xr["delta"], A2, z2(xr["B"]), z2(xr["C"]), xr["dy"], **kw)
    gr = oracle.s6_backward(xr["u"], xr["delta"], xr["A"], xr["B"], xr["C"], xr["dy"], **kw)
    for k in ("du", "ddelta", "dz", "dD", "ddelta_bias"):
        err = max(err, normwise(g[k], gr[k]))
    err = max(err, normwise(g["dA"][:, :N], gr["dA"]))
    for k in ("dB", "dC"):
        err = max(err, normwise(g[k][:, :N], gr[k]))
    return err, 1e-13


def pin_cplx_zoh_expm(lib=None):
    """Each complex state as the real 2-state system [[a, -b], [b, a]] with
    input (Re B, Im B), discretized per step by scipy's matrix exponential of
    the augmented matrix (Van Loan), and read out as Re(C h)."""
    x = make_cplx_inputs(1, 2, 17, 3, seed=92)
    N = 3
    y, last = oracle.s6_cplx_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                     x["D"], x["z"], lib=lib)
    u, dl, z = (_np(x[k])[0] for k in ("u", "delta", "z"))
    A, B, C = _np(x["A"]), _np(x["B"])[0], _np(x["C"])[0]
    bias, D = _np(x["delta_bias"]), _np(x["D"])
    ref = np.empty((2, 17))
    for d in range(2):
        h = np.zeros((N, 2))
        for t in range(17):
            Delta = _softplus(dl[d, t] + bias[d])
            y0 = D[d] * u[d, t]
            for n in range(N):
                a, b = A[d, n], A[d, N + n]
                M = np.zeros((3, 3))
                M[:2, :2] = [[a, -b], [b, a]]
                M[:2, 2] = [B[n, t], B[N + n, t]]
                E = scipy.linalg.expm(Delta * M)
                h[n] = E[:2, :2] @ h[n] + E[:2, 2] * u[d, t]
                y0 += C[n, t] * h[n, 0] - C[N + n, t] * h[n, 1]
            ref[d, t] = y0 * z[d, t] * scipy.special.expit(z[d, t])
    return normwise(y[0], ref), 1e-12


def pin_cplx_held_input_exact(lib=None):
    """u = 1, B = 1, C = 1 (complex ones), time-varying Delta: for a held
    input the zero-order hold is exact, so each complex state is the ODE
    solution h_n(t) = (exp(A_n T_t) - 1) / A_n with T_t = sum_{j<=t} Delta_j,
    and y_t = Re(sum_n h_n(t)); numpy's complex exp on the closed form."""
    N, L = 5, 120
    x = make_inputs(1, 2, L, N, seed=304, has_z=False, has_D=False)
    Ac = np.array([[-0.5 + 1j * n for n in range(N)], [-1.5 + 0.3j * n - 0.2j for n in range(N)]])
    A = np.concatenate([Ac.real, Ac.imag], axis=1)
    ones = np.concatenate([np.ones((1, N, L)), np.zeros((1, N, L))], axis=1)
    y, last = oracle.s6_cplx_forward(np.ones((1, 2, L)), x["delta"], A, ones, ones,
                                     x["delta_bias"], lib=lib)
    Delta = _softplus(_np(x["delta"])[0] + _np(x["delta_bias"])[:, None])
    T = np.cumsum(Delta, axis=1)  # (dim, L)
    h = (np.exp(Ac[:, :, None] * T[:, None, :]) - 1.0) / Ac[:, :, None]  # (dim, N, L)
    ref_last = np.concatenate([h[:, :, -1].real, h[:, :, -1].imag], axis=1)
    return max(normwise(y[0], h.sum(axis=1).real), normwise(last[0], ref_last)), 1e-12


def _cplx_fd_inputs():
    x = make_cplx_inputs(1, 2, 9, 2, seed=93, with_dy=True)
    return {k: (v.double() if v is not None else None) for k, v in x.items()}


def _cplx_loss(x, lib):
    y, _ = oracle.s6_cplx_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                                  x["D"], x["z"], lib=lib, nthreads=1)
    return float(np.sum(_np(x["dy"]) * y))


def pin_cplx_finite_differences(lib=None):
    """Central differences of sum(dy * y) over every real input, including
    the real and imaginary parts of A, B and C."""
    x = _cplx_fd_inputs()
    g = oracle.s6_cplx_backward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"],
                                x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    worst = 0.0
    for name, gname in _GRAD_NAMES.items():
        flat = x[name].reshape(-1)
        fd = np.empty(x[name].shape)
        for i in range(flat.numel()):
            v = float(flat[i])
            h = 1e-6 * max(1.0, abs(v))
            flat[i] = v + h
            lp = _cplx_loss(x, lib)
            flat[i] = v - h
            lm = _cplx_loss(x, lib)
            flat[i] = v
            fd.reshape(-1)[i] = (lp - lm) / (2.0 * h)
        worst = max(worst, normwise(g[gname], fd))
    return worst, 1e-6


def pin_cplx_autograd(lib=None):
    """The complex adjoint against torch.autograd of an independent complex128
    forward (torch's gradient of a complex leaf under a real loss is
    d/d re + i d/d im, the oracle's convention)."""
    x = _cplx_fd_inputs()
    N = x["A"].shape[1] // 2
    to_c = lambda t: torch.complex(t[..., :N, :], t[..., N:, :]) if t.dim() == 3 else \
        torch.complex(t[:, :N], t[:, N:])
    Ac, Bc, Cc = to_c(x["A"]).requires_grad_(True), to_c(x["B"]).requires_grad_(True), \
        to_c(x["C"]).requires_grad_(True)
    leaves = {k: x[k].clone().requires_grad_(True) for k in ("u", "delta", "z", "D", "delta_bias")}
    u, dl, z, D, bias = (leaves[k] for k in ("u", "delta", "z", "D", "delta_bias"))
    Delta = torch.nn.functional.softplus(dl + bias[None, :, None], beta=1.0, threshold=1e9)
    h = torch.zeros(u.shape[0], u.shape[1], N, dtype=torch.complex128)
    ys = []
    for t in range(u.shape[2]):
        xa = Delta[:, :, t, None] * Ac[None]
        Abar = torch.exp(xa)
        Bbar = (Abar - 1.0) / Ac[None] * Bc[:, None, :, t]
        h = Abar * h + Bbar * u[:, :, t, None]
        y0 = (h * Cc[:, None, :, t]).sum(-1).real + D[None] * u[:, :, t]
        ys.append(y0 * torch.nn.functional.silu(z[:, :, t]))
    (torch.stack(ys, dim=-1) * x["dy"]).sum().backward()
    g = oracle.s6_cplx_backward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"],
                                x["delta_bias"], x["D"], x["z"], lib=lib, nthreads=1)
    planar = lambda c, axis: torch.cat([c.real, c.imag], dim=axis).numpy()
    worst = max(normwise(g["dA"], planar(Ac.grad, 1)), normwise(g["dB"], planar(Bc.grad, 1)),
                normwise(g["dC"], planar(Cc.grad, 1)))
    for k, gk in (("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("D", "dD"),
                  ("delta_bias", "ddelta_bias")):
        worst = max(worst, normwise(g[gk], leaves[k].grad.numpy()))
    return worst, 1e-10


ALL_PINS = [pin_golden, pin_theorem1, pin_zoh_expm, pin_lti_convolution, pin_brute_force,
            pin_held_input_exact, pin_skip_and_gate, pin_large_delta_limit,
            pin_small_delta_limit, pin_structure, pin_finite_differences, pin_autograd,
            pin_threads_agree, pin_resume_from_state, pin_initial_state_decay,
            pin_conv_numpy, pin_conv_special_filters, pin_conv_finite_differences,
            pin_conv_autograd, pin_dtproj_matmul, pin_dtproj_finite_differences,
            pin_dtproj_autograd, pin_cplx_real_case, pin_cplx_zoh_expm, pin_cplx_held_input_exact,
            pin_cplx_finite_differences, pin_cplx_autograd]


def run_all(lib=None):
    out = {}
    for fn in ALL_PINS:
        try:
            out[fn.__name__] = fn(lib)
        except Exception as e:  # a broken oracle may also fail by raising
            out[fn.__name__] = (float("inf"), 0.0, repr(e))
    return out
