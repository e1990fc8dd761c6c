"""fp64 CPU oracle for the selective scan (S6) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (the CUDA library and its binding) shares no code with it.

The arithmetic lives in ``s6_oracle.c`` (plain C, fp64, one sequential loop per
(batch, channel)); this module compiles it with gcc on demand and marshals
numpy arrays through ctypes.  See the header of ``s6_oracle.c`` for the pages
and passages each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s6_oracle.c")
_LIB = os.path.join(_HERE, "libs6oracle.so")
_lock = threading.Lock()
_lib = None


def compile_source(src: str, out: str) -> str:
    """Compile one oracle source file into a shared library (gcc, -O2, no
    fast-math, no FMA contraction)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
         "-std=c11", "-pthread", src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``s6_oracle.c`` into ``libs6oracle.so`` if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def load_library(path: str):
    """Load an oracle shared library and declare its entry points."""
    lib = ctypes.CDLL(path)
    dp = ctypes.c_void_p
    i64 = ctypes.c_longlong
    lib.s6_oracle_fwd.argtypes = [dp] * 11 + [i64] * 5
    lib.s6_oracle_fwd.restype = ctypes.c_int
    lib.s6_oracle_bwd.argtypes = [dp] * 17 + [i64] * 5
    lib.s6_oracle_bwd.restype = ctypes.c_int
    lib.s6_oracle_conv_silu.argtypes = [dp] * 3 + [i64] + [dp] * 2 + [i64] * 3
    lib.s6_oracle_conv_silu.restype = ctypes.c_int
    lib.s6_oracle_conv_fwd.argtypes = [dp] * 3 + [i64] + [dp] * 9 + [i64] * 5
    lib.s6_oracle_conv_fwd.restype = ctypes.c_int
    lib.s6_oracle_conv_bwd.argtypes = [dp] * 3 + [i64] + [dp] * 18 + [i64] * 5
    lib.s6_oracle_conv_bwd.restype = ctypes.c_int
    lib.s6_oracle_dtproj_fwd.argtypes = [dp] * 3 + [i64] + [dp] * 8 + [i64] * 5
    lib.s6_oracle_dtproj_fwd.restype = ctypes.c_int
    lib.s6_oracle_dtproj_bwd.argtypes = [dp] * 3 + [i64] + [dp] * 16 + [i64] * 5
    lib.s6_oracle_dtproj_bwd.restype = ctypes.c_int
    lib.s6_oracle_cplx_fwd.argtypes = [dp] * 10 + [i64] * 5
    lib.s6_oracle_cplx_fwd.restype = ctypes.c_int
    lib.s6_oracle_cplx_bwd.argtypes = [dp] * 17 + [i64] * 5
    lib.s6_oracle_cplx_bwd.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load_library(_LIB)
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> exact upcast on the CPU
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def s6_forward(u, delta, A, B, C, delta_bias=None, D=None, z=None, nthreads=None, lib=None,
               initial_state=None):
    """fp64 forward.  Shapes: u, delta, z (batch, dim, L); B, C (batch, N, L);
    A (dim, N); delta_bias, D (dim,); initial_state (batch, dim, N), the state
    before the first step (None = 0).  Returns (y, last_state) as float64
    arrays of shapes (batch, dim, L) and (batch, dim, N)."""
    u, delta, A, B, C = (_f64(t) for t in (u, delta, A, B, C))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    h0 = _f64(initial_state)
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and B.shape == (batch, N, L) and C.shape == (batch, N, L)
    assert A.shape == (dim, N)
    y = np.empty((batch, dim, L), np.float64)
    last = np.empty((batch, dim, N), np.float64)
    rc = (lib or _load()).s6_oracle_fwd(
        _ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(h0), _ptr(y), _ptr(last), batch, dim, L, N, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_fwd failed ({rc})")
    return y, last


def s6_backward(u, delta, A, B, C, dy, delta_bias=None, D=None, z=None, nthreads=None,
                lib=None):
    """fp64 backward of sum(dy * y).  Returns a dict with du, ddelta, dA, dB,
    dC and, when the matching input is given, dD, dz, ddelta_bias."""
    u, delta, A, B, C, dy = (_f64(t) for t in (u, delta, A, B, C, dy))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    batch, dim, L = u.shape
    N = A.shape[1]
    du = np.empty_like(u)
    ddelta = np.empty_like(u)
    dz = np.empty_like(u) if z is not None else None
    dA = np.empty((dim, N), np.float64)
    dB = np.empty((batch, N, L), np.float64)
    dC = np.empty((batch, N, L), np.float64)
    dD = np.empty((dim,), np.float64) if D is not None else None
    dbias = np.empty((dim,), np.float64)
    rc = (lib or _load()).s6_oracle_bwd(
        _ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(dy), _ptr(du), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz),
        _ptr(dbias), batch, dim, L, N, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_bwd failed ({rc})")
    out = {"du": du, "ddelta": ddelta, "dA": dA, "dB": dB, "dC": dC, "ddelta_bias": dbias}
    if dD is not None:
        out["dD"] = dD
    if dz is not None:
        out["dz"] = dz
    return out


def conv_silu(x, conv_w, conv_b=None, lib=None):
    """The convolution prologue alone: returns (pre, u) with
    pre[b,d,t] = conv_b[d] + sum_k conv_w[d,k] x[b,d,t-(W-1)+k] (x = 0 before
    t = 0) and u = SiLU(pre).  x (batch, dim, L); conv_w (dim, W); conv_b
    (dim,) or None."""
    x, conv_w, conv_b = _f64(x), _f64(conv_w), _f64(conv_b)
    batch, dim, L = x.shape
    W = conv_w.shape[1]
    assert conv_w.shape == (dim, W)
    pre = np.empty_like(x)
    u = np.empty_like(x)
    rc = (lib or _load()).s6_oracle_conv_silu(_ptr(x), _ptr(conv_w), _ptr(conv_b), W, _ptr(pre),
                                              _ptr(u), batch, dim, L)
    if rc != 0:
        raise RuntimeError(f"s6_oracle_conv_silu failed ({rc})")
    return pre, u


def s6_conv_forward(x, conv_w, conv_b, delta, A, B, C, delta_bias=None, D=None, z=None,
                    nthreads=None, lib=None):
    """fp64 forward with the convolution prologue: u = SiLU(causal depthwise
    conv of x), then the S6 forward.  Returns (y, last_state)."""
    x, conv_w, conv_b = _f64(x), _f64(conv_w), _f64(conv_b)
    delta, A, B, C = (_f64(t) for t in (delta, A, B, C))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    batch, dim, L = x.shape
    N = A.shape[1]
    W = conv_w.shape[1]
    assert conv_w.shape == (dim, W) and delta.shape == x.shape and B.shape == (batch, N, L)
    y = np.empty((batch, dim, L), np.float64)
    last = np.empty((batch, dim, N), np.float64)
    rc = (lib or _load()).s6_oracle_conv_fwd(
        _ptr(x), _ptr(conv_w), _ptr(conv_b), W, _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(y), _ptr(last), batch, dim, L, N,
        nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_conv_fwd failed ({rc})")
    return y, last


def s6_conv_backward(x, conv_w, conv_b, delta, A, B, C, dy, delta_bias=None, D=None, z=None,
                     nthreads=None, lib=None):
    """fp64 backward of sum(dy * y) for the forward with the convolution
    prologue.  Returns a dict with dx, dconv_w, ddelta, dA, dB, dC,
    ddelta_bias and, when the matching input is given, dconv_b, dD, dz."""
    x, conv_w, conv_b = _f64(x), _f64(conv_w), _f64(conv_b)
    delta, A, B, C, dy = (_f64(t) for t in (delta, A, B, C, dy))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    batch, dim, L = x.shape
    N = A.shape[1]
    W = conv_w.shape[1]
    dx = np.empty_like(x)
    ddelta = np.empty_like(x)
    dz = np.empty_like(x) if z is not None else None
    dcw = np.empty((dim, W), np.float64)
    dcb = np.empty((dim,), np.float64) if conv_b is not None else None
    dA = np.empty((dim, N), np.float64)
    dB = np.empty((batch, N, L), np.float64)
    dC = np.empty((batch, N, L), np.float64)
    dD = np.empty((dim,), np.float64) if D is not None else None
    dbias = np.empty((dim,), np.float64)
    rc = (lib or _load()).s6_oracle_conv_bwd(
        _ptr(x), _ptr(conv_w), _ptr(conv_b), W, _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(dy), _ptr(dx), _ptr(dcw), _ptr(dcb), _ptr(ddelta),
        _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz), _ptr(dbias), batch, dim, L, N,
        nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_conv_bwd failed ({rc})")
    out = {"dx": dx, "dconv_w": dcw, "ddelta": ddelta, "dA": dA, "dB": dB, "dC": dC,
           "ddelta_bias": dbias}
    if dcb is not None:
        out["dconv_b"] = dcb
    if dD is not None:
        out["dD"] = dD
    if dz is not None:
        out["dz"] = dz
    return out


def s6_dtproj_forward(u, dt_low, W_dt, A, B, C, delta_bias=None, D=None, z=None, nthreads=None,
                      lib=None):
    """fp64 forward with the low-rank Delta projection: delta = W_dt . dt_low
    per batch row, then the S6 forward.  dt_low (batch, R, L); W_dt (dim, R).
    Returns (y, last_state)."""
    u, dt_low, W_dt, A, B, C = (_f64(t) for t in (u, dt_low, W_dt, A, B, C))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    batch, dim, L = u.shape
    N = A.shape[1]
    R = W_dt.shape[1]
    assert W_dt.shape == (dim, R) and dt_low.shape == (batch, R, L)
    y = np.empty((batch, dim, L), np.float64)
    last = np.empty((batch, dim, N), np.float64)
    rc = (lib or _load()).s6_oracle_dtproj_fwd(
        _ptr(u), _ptr(dt_low), _ptr(W_dt), R, _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C),
        _ptr(D), _ptr(z), _ptr(y), _ptr(last), batch, dim, L, N, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_dtproj_fwd failed ({rc})")
    return y, last


def s6_dtproj_backward(u, dt_low, W_dt, A, B, C, dy, delta_bias=None, D=None, z=None,
                       nthreads=None, lib=None):
    """fp64 backward of sum(dy * y) for the forward with the projection.
    Returns a dict with du, d_dt_low, dW_dt, dA, dB, dC, ddelta_bias and, when
    the matching input is given, dD, dz."""
    u, dt_low, W_dt, A, B, C, dy = (_f64(t) for t in (u, dt_low, W_dt, A, B, C, dy))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    batch, dim, L = u.shape
    N = A.shape[1]
    R = W_dt.shape[1]
    du = np.empty_like(u)
    dz = np.empty_like(u) if z is not None else None
    ddl = np.empty((batch, R, L), np.float64)
    dW = np.empty((dim, R), np.float64)
    dA = np.empty((dim, N), np.float64)
    dB = np.empty((batch, N, L), np.float64)
    dC = np.empty((batch, N, L), np.float64)
    dD = np.empty((dim,), np.float64) if D is not None else None
    dbias = np.empty((dim,), np.float64)
    rc = (lib or _load()).s6_oracle_dtproj_bwd(
        _ptr(u), _ptr(dt_low), _ptr(W_dt), R, _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C),
        _ptr(D), _ptr(z), _ptr(dy), _ptr(du), _ptr(ddl), _ptr(dW), _ptr(dA), _ptr(dB), _ptr(dC),
        _ptr(dD), _ptr(dz), _ptr(dbias), batch, dim, L, N, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_dtproj_bwd failed ({rc})")
    out = {"du": du, "d_dt_low": ddl, "dW_dt": dW, "dA": dA, "dB": dB, "dC": dC,
           "ddelta_bias": dbias}
    if dD is not None:
        out["dD"] = dD
    if dz is not None:
        out["dz"] = dz
    return out


def s6_cplx_forward(u, delta, A, B, C, delta_bias=None, D=None, z=None, nthreads=None, lib=None):
    """fp64 forward with a complex diagonal A (and complex B, C, state).
    Complex vectors are planar, real parts first: A (dim, 2N); B, C (batch,
    2N, L).  Returns (y (batch, dim, L), last_state (batch, dim, 2N))."""
    u, delta, A, B, C = (_f64(t) for t in (u, delta, A, B, C))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    batch, dim, L = u.shape
    N = A.shape[1] // 2
    assert A.shape == (dim, 2 * N) and B.shape == (batch, 2 * N, L) and C.shape == B.shape
    y = np.empty((batch, dim, L), np.float64)
    last = np.empty((batch, dim, 2 * N), np.float64)
    rc = (lib or _load()).s6_oracle_cplx_fwd(
        _ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(y), _ptr(last), batch, dim, L, N, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_cplx_fwd failed ({rc})")
    return y, last


def s6_cplx_backward(u, delta, A, B, C, dy, delta_bias=None, D=None, z=None, nthreads=None,
                     lib=None):
    """fp64 backward of sum(dy * y) for the complex forward.  Gradients of
    complex inputs are (d/d re, d/d im) pairs in the planar layout.  Returns
    a dict with du, ddelta, dA, dB, dC, ddelta_bias and, when given, dD, dz."""
    u, delta, A, B, C, dy = (_f64(t) for t in (u, delta, A, B, C, dy))
    delta_bias, D, z = _f64(delta_bias), _f64(D), _f64(z)
    batch, dim, L = u.shape
    N = A.shape[1] // 2
    du = np.empty_like(u)
    ddelta = np.empty_like(u)
    dz = np.empty_like(u) if z is not None else None
    dA = np.empty((dim, 2 * N), np.float64)
    dB = np.empty((batch, 2 * N, L), np.float64)
    dC = np.empty((batch, 2 * N, L), np.float64)
    dD = np.empty((dim,), np.float64) if D is not None else None
    dbias = np.empty((dim,), np.float64)
    rc = (lib or _load()).s6_oracle_cplx_bwd(
        _ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(dy), _ptr(du), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(dz),
        _ptr(dbias), batch, dim, L, N, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"s6_oracle_cplx_bwd failed ({rc})")
    out = {"du": du, "ddelta": ddelta, "dA": dA, "dB": dB, "dC": dC, "ddelta_bias": dbias}
    if dD is not None:
        out["dD"] = dD
    if dz is not None:
        out["dz"] = dz
    return out
