"""Python binding of libmambascan (ctypes).  Argument marshalling only: every
step of the selective scan runs in the library's CUDA kernels.  There is no
CPU fallback; a missing library or device raises.

Low-level calls (same names and argument order as ``include/mamba_scan.h``):
``mamba_scan_fwd``, ``mamba_scan_bwd``, ``mamba_conv_scan_fwd``,
``mamba_conv_scan_bwd``, ``mamba_dtproj_scan_fwd``, ``mamba_dtproj_scan_bwd``
(with the training pairs ``*_saved_bytes`` / ``*_fwd_save`` / ``*_bwd_saved``),
``mamba_cplx_scan_fwd``, ``mamba_cplx_scan_bwd``, ``mamba_scan_step``,
``mamba_scan_fwd_noalloc``,
``mamba_scan_stream_status``; decoding plans (``StepPlan``), the workspace
pool (``pool_set_reserve``, ``pool_trim``, ``pool_reserved``) and the
allocation-failure test hook (``test_fail_alloc``).  Convenience wrappers that allocate the outputs:
``selective_scan_fwd``, ``selective_scan_bwd``, ``conv_selective_scan_fwd``
and ``conv_selective_scan_bwd``.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

# MAMBA_SCAN_LIBRARY selects another build of the same library (the
# bounds-checking libmambascan_debug.so, for the tests that run against it).
_LIB_PATH = os.environ.get("MAMBA_SCAN_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "lib", "libmambascan.so")

MAMBA_F32, MAMBA_BF16 = 0, 1
PATH_AUTO, PATH_REFERENCE, PATH_GENERIC, PATH_STRUCTURED = 0, 1, 2, 3
PATHS = {"auto": PATH_AUTO, "reference": PATH_REFERENCE, "generic": PATH_GENERIC,
         "structured": PATH_STRUCTURED}
STATUS = {0: "MAMBA_OK", 1: "MAMBA_ERR_INVALID_ARG", 2: "MAMBA_ERR_UNSUPPORTED",
          3: "MAMBA_ERR_CUDA", 4: "MAMBA_ERR_OUT_OF_MEMORY", 5: "MAMBA_ERR_DEVICE_TIMEOUT",
          6: "MAMBA_ERR_OUT_OF_BOUNDS"}


class MambaScanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class _Options(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
                ("carry", ctypes.c_int32), ("wait_timeout_us", ctypes.c_int32),
                ("test_hook", ctypes.c_int32), ("reserved", ctypes.c_int32 * 3)]


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libmambascan.so (built in-tree by ``selective_state_space_21_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"libmambascan.so not found at {_LIB_PATH}; build it with "
                    "`python -m selective_state_space_21_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            opt = ctypes.POINTER(_Options)
            lib.mamba_scan_fwd.argtypes = [vp] * 10 + [i64] * 4 + [i32, vp]
            lib.mamba_scan_fwd_ex.argtypes = [vp] * 10 + [i64] * 4 + [i32, opt, vp]
            lib.mamba_scan_bwd.argtypes = [vp] * 17 + [i64] * 4 + [i32, vp]
            lib.mamba_scan_bwd_ex.argtypes = [vp] * 17 + [i64] * 4 + [i32, opt, vp]
            lib.mamba_scan_fwd_noalloc.argtypes = [vp] * 10 + [i64] * 4 + [i32, vp]
            u64 = ctypes.c_uint64
            lib.mamba_scan_saved_bytes.argtypes = [i64] * 4 + [i32, opt, ctypes.POINTER(u64)]
            lib.mamba_scan_saved_bytes.restype = ctypes.c_int
            lib.mamba_scan_fwd_save.argtypes = [vp] * 10 + [i64] * 4 + [i32, opt, vp, u64, vp]
            lib.mamba_scan_fwd_save.restype = ctypes.c_int
            lib.mamba_scan_bwd_saved.argtypes = [vp] * 17 + [i64] * 4 + [i32, opt, vp, u64, vp]
            lib.mamba_scan_bwd_saved.restype = ctypes.c_int
            lib.mamba_conv_scan_saved_bytes.argtypes = [i64] * 5 + [i32, opt, ctypes.POINTER(u64)]
            lib.mamba_conv_scan_saved_bytes.restype = ctypes.c_int
            lib.mamba_conv_scan_fwd_save.argtypes = (
                [vp] * 3 + [i64] + [vp] * 9 + [i64] * 4 + [i32, opt, vp, u64, vp])
            lib.mamba_conv_scan_fwd_save.restype = ctypes.c_int
            lib.mamba_conv_scan_bwd_saved.argtypes = (
                [vp] * 3 + [i64] + [vp] * 18 + [i64] * 4 + [i32, opt, vp, u64, vp])
            lib.mamba_conv_scan_bwd_saved.restype = ctypes.c_int
            lib.mamba_scan_step.argtypes = [vp] * 10 + [i64] * 3 + [i32, vp]
            lib.mamba_scan_step.restype = ctypes.c_int
            lib.mamba_conv_scan_step.argtypes = [vp] * 5 + [i64] + [vp] * 8 + [i64] * 3 + [i32, vp]
            lib.mamba_conv_scan_step.restype = ctypes.c_int
            lib.mamba_conv_scan_fwd.argtypes = [vp] * 3 + [i64] + [vp] * 9 + [i64] * 4 + [i32, opt, vp]
            lib.mamba_conv_scan_fwd.restype = ctypes.c_int
            lib.mamba_conv_scan_bwd.argtypes = [vp] * 3 + [i64] + [vp] * 18 + [i64] * 4 + [i32, opt, vp]
            lib.mamba_conv_scan_bwd.restype = ctypes.c_int
            lib.mamba_dtproj_scan_fwd.argtypes = [vp] * 3 + [i64] + [vp] * 8 + [i64] * 4 + [i32, opt, vp]
            lib.mamba_dtproj_scan_fwd.restype = ctypes.c_int
            lib.mamba_dtproj_scan_bwd.argtypes = [vp] * 3 + [i64] + [vp] * 16 + [i64] * 4 + [i32, opt, vp]
            lib.mamba_dtproj_scan_bwd.restype = ctypes.c_int
            lib.mamba_dtproj_scan_saved_bytes.argtypes = [i64] * 5 + [i32, opt, ctypes.POINTER(u64)]
            lib.mamba_dtproj_scan_saved_bytes.restype = ctypes.c_int
            lib.mamba_dtproj_scan_fwd_save.argtypes = (
                [vp] * 3 + [i64] + [vp] * 8 + [i64] * 4 + [i32, opt, vp, u64, vp])
            lib.mamba_dtproj_scan_fwd_save.restype = ctypes.c_int
            lib.mamba_dtproj_scan_bwd_saved.argtypes = (
                [vp] * 3 + [i64] + [vp] * 16 + [i64] * 4 + [i32, opt, vp, u64, vp])
            lib.mamba_dtproj_scan_bwd_saved.restype = ctypes.c_int
            lib.mamba_cplx_scan_fwd.argtypes = [vp] * 10 + [i64] * 4 + [i32, vp]
            lib.mamba_cplx_scan_fwd.restype = ctypes.c_int
            lib.mamba_cplx_scan_bwd.argtypes = [vp] * 17 + [i64] * 4 + [i32, vp]
            lib.mamba_cplx_scan_bwd.restype = ctypes.c_int
            lib.mamba_cplx_scan_saved_bytes.argtypes = [i64] * 4 + [i32, ctypes.POINTER(ctypes.c_uint64)]
            lib.mamba_cplx_scan_saved_bytes.restype = ctypes.c_int
            lib.mamba_cplx_scan_fwd_save.argtypes = [vp] * 10 + [i64] * 4 + [i32, vp, ctypes.c_uint64, vp]
            lib.mamba_cplx_scan_fwd_save.restype = ctypes.c_int
            lib.mamba_cplx_scan_bwd_saved.argtypes = [vp] * 17 + [i64] * 4 + [i32, vp, ctypes.c_uint64, vp]
            lib.mamba_cplx_scan_bwd_saved.restype = ctypes.c_int
            for f in ("mamba_scan_fwd", "mamba_scan_fwd_ex", "mamba_scan_bwd",
                      "mamba_scan_bwd_ex", "mamba_scan_stream_status", "mamba_scan_fwd_noalloc"):
                getattr(lib, f).restype = ctypes.c_int
            lib.mamba_scan_stream_status.argtypes = [vp]
            lib.mamba_scan_status_string.argtypes = [ctypes.c_int]
            lib.mamba_scan_status_string.restype = ctypes.c_char_p
            lib.mamba_scan_launch_count.argtypes = []
            lib.mamba_scan_launch_count.restype = ctypes.c_uint64
            lib.mamba_scan_abi_version.argtypes = []
            lib.mamba_scan_abi_version.restype = ctypes.c_int
            lib.mamba_scan_step_plan_create.argtypes = (
                [ctypes.POINTER(vp)] + [vp] * 5 + [i64] + [vp] * 8 + [i64] * 3 + [i32])
            lib.mamba_scan_step_plan_create.restype = ctypes.c_int
            lib.mamba_scan_step_plan_run.argtypes = [vp, vp]
            lib.mamba_scan_step_plan_run.restype = ctypes.c_int
            lib.mamba_scan_step_plan_destroy.argtypes = [vp]
            lib.mamba_scan_step_plan_destroy.restype = None
            lib.mamba_scan_pool_set_reserve.argtypes = [ctypes.c_uint64]
            lib.mamba_scan_pool_set_reserve.restype = ctypes.c_int
            lib.mamba_scan_pool_trim.argtypes = [ctypes.c_uint64]
            lib.mamba_scan_pool_trim.restype = ctypes.c_int
            lib.mamba_scan_pool_reserved.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
            lib.mamba_scan_pool_reserved.restype = ctypes.c_int
            lib.mamba_scan_test_fail_alloc.argtypes = [ctypes.c_int32]
            lib.mamba_scan_test_fail_alloc.restype = None
            _lib = lib
    return _lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return MAMBA_F32
    if t == torch.bfloat16:
        return MAMBA_BF16
    raise TypeError(f"unsupported I/O dtype {t} (float32 or bfloat16)")


def _ptr(t: Optional[torch.Tensor], dtype=None, shape=None, name=""):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr() if t.numel() > 0 else None


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        # torch's current stream of the current device, without building a
        # Stream object per call (it matters for one-token decoding steps)
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:
            return raw(torch.cuda.current_device())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


CARRY = {"auto": 0, "sequential": 1, "three_phase": 2}


def _options(path, chunk_len, carry="auto", wait_timeout_us=0, test_hook=0):
    o = _Options()
    o.path = PATHS[path] if isinstance(path, str) else int(path)
    o.chunk_len = int(chunk_len)
    o.carry = CARRY[carry] if isinstance(carry, str) else int(carry)
    o.wait_timeout_us = int(wait_timeout_us)
    o.test_hook = int(test_hook)
    return o


def _check(rc: int, where: str):
    if rc != 0:
        raise MambaScanError(rc, where)


def mamba_scan_fwd(u, delta, delta_bias, A, B, C, D, z, y, last_state, *, path="auto",
                   chunk_len=0, carry="auto", wait_timeout_us=0, test_hook=0, stream=None):
    """Enqueue the forward on ``stream`` (torch's current stream by default).
    Tensors as in ``include/mamba_scan.h``; ``y`` (and ``last_state``) are
    written."""
    batch, dim, L = u.shape
    N = A.shape[1]
    dt = u.dtype
    f32 = torch.float32
    args = [
        _ptr(u, dt, (batch, dim, L), "u"), _ptr(delta, dt, (batch, dim, L), "delta"),
        _ptr(delta_bias, f32, (dim,), "delta_bias"), _ptr(A, f32, (dim, N), "A"),
        _ptr(B, dt, (batch, N, L), "B"), _ptr(C, dt, (batch, N, L), "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, (batch, dim, L), "z"),
        _ptr(y, dt, (batch, dim, L), "y"), _ptr(last_state, f32, (batch, dim, N), "last_state"),
        batch, dim, L, N, _dtype_code(dt)]
    lib = load_library()
    if path == "auto" and not chunk_len and carry == "auto" and not wait_timeout_us \
            and not test_hook:
        rc = lib.mamba_scan_fwd(*args, _stream_handle(stream))
    else:
        opts = _options(path, chunk_len, carry, wait_timeout_us, test_hook)
        rc = lib.mamba_scan_fwd_ex(*args, ctypes.byref(opts), _stream_handle(stream))
    _check(rc, "mamba_scan_fwd")


def mamba_scan_bwd(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                   ddelta_bias, *, path="auto", chunk_len=0, carry="auto", wait_timeout_us=0,
                   test_hook=0, stream=None):
    """Enqueue the backward of sum(dy * y) on ``stream``; the gradient tensors
    are written."""
    batch, dim, L = u.shape
    N = A.shape[1]
    dt = u.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, N, L)
    args = [
        _ptr(u, dt, bdl, "u"), _ptr(delta, dt, bdl, "delta"),
        _ptr(delta_bias, f32, (dim,), "delta_bias"), _ptr(A, f32, (dim, N), "A"),
        _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"), _ptr(D, f32, (dim,), "D"),
        _ptr(z, dt, bdl, "z"), _ptr(dy, dt, bdl, "dy"), _ptr(du, dt, bdl, "du"),
        _ptr(ddelta, dt, bdl, "ddelta"), _ptr(dA, f32, (dim, N), "dA"),
        _ptr(dB, dt, bnl, "dB"), _ptr(dC, dt, bnl, "dC"), _ptr(dD, f32, (dim,), "dD"),
        _ptr(dz, dt, bdl, "dz"), _ptr(ddelta_bias, f32, (dim,), "ddelta_bias"),
        batch, dim, L, N, _dtype_code(dt)]
    lib = load_library()
    if path == "auto" and not chunk_len and carry == "auto" and not wait_timeout_us \
            and not test_hook:
        rc = lib.mamba_scan_bwd(*args, _stream_handle(stream))
    else:
        opts = _options(path, chunk_len, carry, wait_timeout_us, test_hook)
        rc = lib.mamba_scan_bwd_ex(*args, ctypes.byref(opts), _stream_handle(stream))
    _check(rc, "mamba_scan_bwd")


def saved_bytes(batch, dim, L, N, dtype, *, path="auto", chunk_len=0, carry="auto",
                wait_timeout_us=0, test_hook=0) -> int:
    """Bytes of the buffer the saving forward (``mamba_scan_fwd_save``) fills
    for its backward on the current device; 0 where the problem takes the
    one-thread-per-channel kernels (then the pair is the plain forward and
    backward, and ``saved`` may be None)."""
    n = ctypes.c_uint64(0)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_scan_saved_bytes(batch, dim, L, N, _dtype_code(dtype), opts,
                                                 ctypes.byref(n)), "mamba_scan_saved_bytes")
    return int(n.value)


def _saved_arg(saved, need, name="saved"):
    if need == 0:
        return None, 0
    if saved is None or saved.dtype != torch.uint8:
        raise TypeError(f"{name} must be a uint8 CUDA tensor of at least {need} bytes")
    if saved.numel() < need:
        raise ValueError(f"{name} holds {saved.numel()} bytes; {need} are needed")
    return _ptr(saved, torch.uint8, None, name), saved.numel()


def mamba_scan_fwd_save(u, delta, delta_bias, A, B, C, D, z, y, last_state, saved, *,
                        path="auto", chunk_len=0, carry="auto", wait_timeout_us=0, test_hook=0,
                        stream=None):
    """``mamba_scan_fwd`` that also fills ``saved`` (a uint8 CUDA tensor of
    ``saved_bytes(...)`` bytes) with what ``mamba_scan_bwd_saved`` reads in
    place of re-running the forward."""
    batch, dim, L = u.shape
    N = A.shape[1]
    dt = u.dtype
    f32 = torch.float32
    need = saved_bytes(batch, dim, L, N, dt, path=path, chunk_len=chunk_len, carry=carry,
                       wait_timeout_us=wait_timeout_us, test_hook=test_hook)
    sp, sn = _saved_arg(saved, need)
    args = [
        _ptr(u, dt, (batch, dim, L), "u"), _ptr(delta, dt, (batch, dim, L), "delta"),
        _ptr(delta_bias, f32, (dim,), "delta_bias"), _ptr(A, f32, (dim, N), "A"),
        _ptr(B, dt, (batch, N, L), "B"), _ptr(C, dt, (batch, N, L), "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, (batch, dim, L), "z"),
        _ptr(y, dt, (batch, dim, L), "y"), _ptr(last_state, f32, (batch, dim, N), "last_state"),
        batch, dim, L, N, _dtype_code(dt)]
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_scan_fwd_save(*args, opts, sp, sn, _stream_handle(stream)),
           "mamba_scan_fwd_save")


def mamba_scan_bwd_saved(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                         ddelta_bias, saved, *, path="auto", chunk_len=0, carry="auto",
                         wait_timeout_us=0, test_hook=0, stream=None):
    """``mamba_scan_bwd`` reading ``saved`` as ``mamba_scan_fwd_save`` wrote it
    (same inputs and options) instead of re-running the forward."""
    batch, dim, L = u.shape
    N = A.shape[1]
    dt = u.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, N, L)
    need = saved_bytes(batch, dim, L, N, dt, path=path, chunk_len=chunk_len, carry=carry,
                       wait_timeout_us=wait_timeout_us, test_hook=test_hook)
    sp, sn = _saved_arg(saved, need)
    args = [
        _ptr(u, dt, bdl, "u"), _ptr(delta, dt, bdl, "delta"),
        _ptr(delta_bias, f32, (dim,), "delta_bias"), _ptr(A, f32, (dim, N), "A"),
        _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"), _ptr(D, f32, (dim,), "D"),
        _ptr(z, dt, bdl, "z"), _ptr(dy, dt, bdl, "dy"), _ptr(du, dt, bdl, "du"),
        _ptr(ddelta, dt, bdl, "ddelta"), _ptr(dA, f32, (dim, N), "dA"),
        _ptr(dB, dt, bnl, "dB"), _ptr(dC, dt, bnl, "dC"), _ptr(dD, f32, (dim,), "dD"),
        _ptr(dz, dt, bdl, "dz"), _ptr(ddelta_bias, f32, (dim,), "ddelta_bias"),
        batch, dim, L, N, _dtype_code(dt)]
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_scan_bwd_saved(*args, opts, sp, sn, _stream_handle(stream)),
           "mamba_scan_bwd_saved")


def _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook):
    if path == "auto" and not chunk_len and carry == "auto" and not wait_timeout_us \
            and not test_hook:
        return None
    return ctypes.byref(_options(path, chunk_len, carry, wait_timeout_us, test_hook))


def _conv_fwd_args(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, y, last_state):
    batch, dim, L = x.shape
    N = A.shape[1]
    W = conv_w.shape[1]
    dt = x.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, N, L)
    args = [
        _ptr(x, dt, bdl, "x"), _ptr(conv_w, f32, (dim, W), "conv_w"),
        _ptr(conv_b, f32, (dim,), "conv_b"), W,
        _ptr(delta, dt, bdl, "delta"), _ptr(delta_bias, f32, (dim,), "delta_bias"),
        _ptr(A, f32, (dim, N), "A"), _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, bdl, "z"), _ptr(y, dt, bdl, "y"),
        _ptr(last_state, f32, (batch, dim, N), "last_state"), batch, dim, L, N, _dtype_code(dt)]
    return args


def mamba_conv_scan_fwd(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, y, last_state, *,
                        path="auto", chunk_len=0, carry="auto", wait_timeout_us=0, test_hook=0,
                        stream=None):
    """Enqueue the forward with the convolution prologue (u = SiLU(causal
    depthwise conv of x) computed inside the scan kernels).  x (batch, dim, L)
    in the I/O dtype; conv_w (dim, W) float32 with W in 1..4; conv_b (dim,)
    float32 or None; the rest as ``mamba_scan_fwd``."""
    args = _conv_fwd_args(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, y, last_state)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_conv_scan_fwd(*args, opts, _stream_handle(stream)),
           "mamba_conv_scan_fwd")


def conv_saved_bytes(batch, dim, L, N, conv_width, dtype, *, path="auto", chunk_len=0,
                     carry="auto", wait_timeout_us=0, test_hook=0) -> int:
    """``saved_bytes`` for the training pair with the convolution prologue."""
    n = ctypes.c_uint64(0)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_conv_scan_saved_bytes(batch, dim, L, N, conv_width,
                                                      _dtype_code(dtype), opts, ctypes.byref(n)),
           "mamba_conv_scan_saved_bytes")
    return int(n.value)


def mamba_conv_scan_fwd_save(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, y, last_state,
                             saved, *, path="auto", chunk_len=0, carry="auto", wait_timeout_us=0,
                             test_hook=0, stream=None):
    """``mamba_conv_scan_fwd`` that also fills ``saved`` (``conv_saved_bytes``
    bytes) for ``mamba_conv_scan_bwd_saved``."""
    batch, dim, L = x.shape
    need = conv_saved_bytes(batch, dim, L, A.shape[1], conv_w.shape[1], x.dtype, path=path,
                            chunk_len=chunk_len, carry=carry, wait_timeout_us=wait_timeout_us,
                            test_hook=test_hook)
    sp, sn = _saved_arg(saved, need)
    args = _conv_fwd_args(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, y, last_state)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_conv_scan_fwd_save(*args, opts, sp, sn, _stream_handle(stream)),
           "mamba_conv_scan_fwd_save")


def _conv_bwd_args(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, dy, dx, dconv_w, dconv_b,
                   ddelta, dA, dB, dC, dD, dz, ddelta_bias):
    batch, dim, L = x.shape
    N = A.shape[1]
    W = conv_w.shape[1]
    dt = x.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, N, L)
    args = [
        _ptr(x, dt, bdl, "x"), _ptr(conv_w, f32, (dim, W), "conv_w"),
        _ptr(conv_b, f32, (dim,), "conv_b"), W,
        _ptr(delta, dt, bdl, "delta"), _ptr(delta_bias, f32, (dim,), "delta_bias"),
        _ptr(A, f32, (dim, N), "A"), _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, bdl, "z"), _ptr(dy, dt, bdl, "dy"),
        _ptr(dx, dt, bdl, "dx"), _ptr(dconv_w, f32, (dim, W), "dconv_w"),
        _ptr(dconv_b, f32, (dim,), "dconv_b"), _ptr(ddelta, dt, bdl, "ddelta"),
        _ptr(dA, f32, (dim, N), "dA"), _ptr(dB, dt, bnl, "dB"), _ptr(dC, dt, bnl, "dC"),
        _ptr(dD, f32, (dim,), "dD"), _ptr(dz, dt, bdl, "dz"),
        _ptr(ddelta_bias, f32, (dim,), "ddelta_bias"), batch, dim, L, N, _dtype_code(dt)]
    return args


def mamba_conv_scan_bwd(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, dy, dx, dconv_w,
                        dconv_b, ddelta, dA, dB, dC, dD, dz, ddelta_bias, *, path="auto",
                        chunk_len=0, carry="auto", wait_timeout_us=0, test_hook=0, stream=None):
    """Enqueue the backward of sum(dy * y) for ``mamba_conv_scan_fwd``: dx
    and dconv_w (and dconv_b if given) take the place of du."""
    args = _conv_bwd_args(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, dy, dx, dconv_w,
                          dconv_b, ddelta, dA, dB, dC, dD, dz, ddelta_bias)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_conv_scan_bwd(*args, opts, _stream_handle(stream)),
           "mamba_conv_scan_bwd")


def mamba_conv_scan_bwd_saved(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, dy, dx,
                              dconv_w, dconv_b, ddelta, dA, dB, dC, dD, dz, ddelta_bias, saved, *,
                              path="auto", chunk_len=0, carry="auto", wait_timeout_us=0,
                              test_hook=0, stream=None):
    """``mamba_conv_scan_bwd`` reading ``saved`` as ``mamba_conv_scan_fwd_save``
    wrote it (same inputs and options)."""
    batch, dim, L = x.shape
    need = conv_saved_bytes(batch, dim, L, A.shape[1], conv_w.shape[1], x.dtype, path=path,
                            chunk_len=chunk_len, carry=carry, wait_timeout_us=wait_timeout_us,
                            test_hook=test_hook)
    sp, sn = _saved_arg(saved, need)
    args = _conv_bwd_args(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, dy, dx, dconv_w,
                          dconv_b, ddelta, dA, dB, dC, dD, dz, ddelta_bias)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_conv_scan_bwd_saved(*args, opts, sp, sn, _stream_handle(stream)),
           "mamba_conv_scan_bwd_saved")


def _dtproj_fwd_args(u, dt_low, W_dt, delta_bias, A, B, C, D, z, y, last_state):
    batch, dim, L = u.shape
    N = A.shape[1]
    R = W_dt.shape[1]
    dt = u.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, N, L)
    return [
        _ptr(u, dt, bdl, "u"), _ptr(dt_low, dt, (batch, R, L), "dt_low"),
        _ptr(W_dt, dt, (dim, R), "W_dt"), R, _ptr(delta_bias, f32, (dim,), "delta_bias"),
        _ptr(A, f32, (dim, N), "A"), _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, bdl, "z"), _ptr(y, dt, bdl, "y"),
        _ptr(last_state, f32, (batch, dim, N), "last_state"), batch, dim, L, N, _dtype_code(dt)]


def mamba_dtproj_scan_fwd(u, dt_low, W_dt, delta_bias, A, B, C, D, z, y, last_state, *,
                          path="auto", chunk_len=0, carry="auto", wait_timeout_us=0,
                          test_hook=0, stream=None):
    """Enqueue the forward with the low-rank Delta projection: delta =
    W_dt . dt_low per batch row (a tensor-core GEMM), then the scan.  dt_low
    (batch, R, L) and W_dt (dim, R) in the I/O dtype; the rest as
    ``mamba_scan_fwd``."""
    args = _dtproj_fwd_args(u, dt_low, W_dt, delta_bias, A, B, C, D, z, y, last_state)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_dtproj_scan_fwd(*args, opts, _stream_handle(stream)),
           "mamba_dtproj_scan_fwd")


def dtproj_saved_bytes(batch, dim, L, N, R, dtype, *, path="auto", chunk_len=0, carry="auto",
                       wait_timeout_us=0, test_hook=0) -> int:
    """``saved_bytes`` for the training pair with the Delta projection (0 where
    the pair behaves as the plain calls)."""
    n = ctypes.c_uint64(0)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_dtproj_scan_saved_bytes(batch, dim, L, N, R, _dtype_code(dtype),
                                                        opts, ctypes.byref(n)),
           "mamba_dtproj_scan_saved_bytes")
    return int(n.value)


def mamba_dtproj_scan_fwd_save(u, dt_low, W_dt, delta_bias, A, B, C, D, z, y, last_state, saved,
                               *, path="auto", chunk_len=0, carry="auto", wait_timeout_us=0,
                               test_hook=0, stream=None):
    """``mamba_dtproj_scan_fwd`` that also fills ``saved``
    (``dtproj_saved_bytes`` bytes) for ``mamba_dtproj_scan_bwd_saved``."""
    batch, dim, L = u.shape
    need = dtproj_saved_bytes(batch, dim, L, A.shape[1], W_dt.shape[1], u.dtype, path=path,
                              chunk_len=chunk_len, carry=carry, wait_timeout_us=wait_timeout_us,
                              test_hook=test_hook)
    sp, sn = _saved_arg(saved, need)
    args = _dtproj_fwd_args(u, dt_low, W_dt, delta_bias, A, B, C, D, z, y, last_state)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_dtproj_scan_fwd_save(*args, opts, sp, sn, _stream_handle(stream)),
           "mamba_dtproj_scan_fwd_save")


def _dtproj_bwd_args(u, dt_low, W_dt, delta_bias, A, B, C, D, z, dy, du, d_dt_low, dW_dt, dA, dB,
                     dC, dD, dz, ddelta_bias):
    batch, dim, L = u.shape
    N = A.shape[1]
    R = W_dt.shape[1]
    dt = u.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, N, L)
    return [
        _ptr(u, dt, bdl, "u"), _ptr(dt_low, dt, (batch, R, L), "dt_low"),
        _ptr(W_dt, dt, (dim, R), "W_dt"), R, _ptr(delta_bias, f32, (dim,), "delta_bias"),
        _ptr(A, f32, (dim, N), "A"), _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, bdl, "z"), _ptr(dy, dt, bdl, "dy"),
        _ptr(du, dt, bdl, "du"), _ptr(d_dt_low, dt, (batch, R, L), "d_dt_low"),
        _ptr(dW_dt, f32, (dim, R), "dW_dt"), _ptr(dA, f32, (dim, N), "dA"),
        _ptr(dB, dt, bnl, "dB"), _ptr(dC, dt, bnl, "dC"), _ptr(dD, f32, (dim,), "dD"),
        _ptr(dz, dt, bdl, "dz"), _ptr(ddelta_bias, f32, (dim,), "ddelta_bias"),
        batch, dim, L, N, _dtype_code(dt)]


def mamba_dtproj_scan_bwd(u, dt_low, W_dt, delta_bias, A, B, C, D, z, dy, du, d_dt_low, dW_dt,
                          dA, dB, dC, dD, dz, ddelta_bias, *, path="auto", chunk_len=0,
                          wait_timeout_us=0, test_hook=0, stream=None):
    """Enqueue the backward of sum(dy * y) for ``mamba_dtproj_scan_fwd``:
    d_dt_low (batch, R, L, I/O dtype) and dW_dt (dim, R, float32) take the
    place of ddelta."""
    args = _dtproj_bwd_args(u, dt_low, W_dt, delta_bias, A, B, C, D, z, dy, du, d_dt_low, dW_dt,
                            dA, dB, dC, dD, dz, ddelta_bias)
    opts = _opts_ptr(path, chunk_len, "auto", wait_timeout_us, test_hook)
    _check(load_library().mamba_dtproj_scan_bwd(*args, opts, _stream_handle(stream)),
           "mamba_dtproj_scan_bwd")


def mamba_dtproj_scan_bwd_saved(u, dt_low, W_dt, delta_bias, A, B, C, D, z, dy, du, d_dt_low,
                                dW_dt, dA, dB, dC, dD, dz, ddelta_bias, saved, *, path="auto",
                                chunk_len=0, carry="auto", wait_timeout_us=0, test_hook=0,
                                stream=None):
    """``mamba_dtproj_scan_bwd`` reading ``saved`` as
    ``mamba_dtproj_scan_fwd_save`` wrote it (same inputs and options)."""
    batch, dim, L = u.shape
    need = dtproj_saved_bytes(batch, dim, L, A.shape[1], W_dt.shape[1], u.dtype, path=path,
                              chunk_len=chunk_len, carry=carry, wait_timeout_us=wait_timeout_us,
                              test_hook=test_hook)
    sp, sn = _saved_arg(saved, need)
    args = _dtproj_bwd_args(u, dt_low, W_dt, delta_bias, A, B, C, D, z, dy, du, d_dt_low, dW_dt,
                            dA, dB, dC, dD, dz, ddelta_bias)
    opts = _opts_ptr(path, chunk_len, carry, wait_timeout_us, test_hook)
    _check(load_library().mamba_dtproj_scan_bwd_saved(*args, opts, sp, sn, _stream_handle(stream)),
           "mamba_dtproj_scan_bwd_saved")


def _cplx_fwd_args(u, delta, delta_bias, A, B, C, D, z, y, last_state):
    batch, dim, L = u.shape
    N = A.shape[1] // 2
    dt = u.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, 2 * N, L)
    args = [
        _ptr(u, dt, bdl, "u"), _ptr(delta, dt, bdl, "delta"),
        _ptr(delta_bias, f32, (dim,), "delta_bias"), _ptr(A, f32, (dim, 2 * N), "A"),
        _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"), _ptr(D, f32, (dim,), "D"),
        _ptr(z, dt, bdl, "z"), _ptr(y, dt, bdl, "y"),
        _ptr(last_state, f32, (batch, dim, 2 * N), "last_state"), batch, dim, L, N,
        _dtype_code(dt)]
    return args


def mamba_cplx_scan_fwd(u, delta, delta_bias, A, B, C, D, z, y, last_state, *, stream=None):
    """Enqueue the forward with a complex diagonal A.  Complex vectors are
    planar, real parts first: A (dim, 2N) float32, B and C (batch, 2N, L) in
    the I/O dtype, last_state (batch, dim, 2N) float32."""
    args = _cplx_fwd_args(u, delta, delta_bias, A, B, C, D, z, y, last_state)
    _check(load_library().mamba_cplx_scan_fwd(*args, _stream_handle(stream)),
           "mamba_cplx_scan_fwd")


def cplx_saved_bytes(batch, dim, L, N, dtype) -> int:
    """Bytes of the block checkpoints the complex training pair keeps."""
    n = ctypes.c_uint64(0)
    _check(load_library().mamba_cplx_scan_saved_bytes(batch, dim, L, N, _dtype_code(dtype),
                                                      ctypes.byref(n)),
           "mamba_cplx_scan_saved_bytes")
    return int(n.value)


def mamba_cplx_scan_fwd_save(u, delta, delta_bias, A, B, C, D, z, y, last_state, saved, *,
                             stream=None):
    """``mamba_cplx_scan_fwd`` that also fills ``saved`` (``cplx_saved_bytes``
    bytes, uint8) with the block checkpoints for ``mamba_cplx_scan_bwd_saved``."""
    batch, dim, L = u.shape
    need = cplx_saved_bytes(batch, dim, L, A.shape[1] // 2, u.dtype)
    sp, sn = _saved_arg(saved, need)
    args = _cplx_fwd_args(u, delta, delta_bias, A, B, C, D, z, y, last_state)
    _check(load_library().mamba_cplx_scan_fwd_save(*args, sp, sn, _stream_handle(stream)),
           "mamba_cplx_scan_fwd_save")


def _cplx_bwd_args(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                   ddelta_bias):
    batch, dim, L = u.shape
    N = A.shape[1] // 2
    dt = u.dtype
    f32 = torch.float32
    bdl, bnl = (batch, dim, L), (batch, 2 * N, L)
    args = [
        _ptr(u, dt, bdl, "u"), _ptr(delta, dt, bdl, "delta"),
        _ptr(delta_bias, f32, (dim,), "delta_bias"), _ptr(A, f32, (dim, 2 * N), "A"),
        _ptr(B, dt, bnl, "B"), _ptr(C, dt, bnl, "C"), _ptr(D, f32, (dim,), "D"),
        _ptr(z, dt, bdl, "z"), _ptr(dy, dt, bdl, "dy"), _ptr(du, dt, bdl, "du"),
        _ptr(ddelta, dt, bdl, "ddelta"), _ptr(dA, f32, (dim, 2 * N), "dA"),
        _ptr(dB, dt, bnl, "dB"), _ptr(dC, dt, bnl, "dC"), _ptr(dD, f32, (dim,), "dD"),
        _ptr(dz, dt, bdl, "dz"), _ptr(ddelta_bias, f32, (dim,), "ddelta_bias"),
        batch, dim, L, N, _dtype_code(dt)]
    return args


def mamba_cplx_scan_bwd(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                        ddelta_bias, *, stream=None):
    """Enqueue the backward of sum(dy * y) for ``mamba_cplx_scan_fwd``; dA
    (dim, 2N) float32 and dB, dC (batch, 2N, L) hold (d/d re, d/d im) pairs,
    planar."""
    args = _cplx_bwd_args(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                          ddelta_bias)
    _check(load_library().mamba_cplx_scan_bwd(*args, _stream_handle(stream)),
           "mamba_cplx_scan_bwd")


def mamba_cplx_scan_bwd_saved(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD,
                              dz, ddelta_bias, saved, *, stream=None):
    """``mamba_cplx_scan_bwd`` reading the block checkpoints
    ``mamba_cplx_scan_fwd_save`` stored, in place of its forward sweep."""
    batch, dim, L = u.shape
    need = cplx_saved_bytes(batch, dim, L, A.shape[1] // 2, u.dtype)
    sp, sn = _saved_arg(saved, need)
    args = _cplx_bwd_args(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                          ddelta_bias)
    _check(load_library().mamba_cplx_scan_bwd_saved(*args, sp, sn, _stream_handle(stream)),
           "mamba_cplx_scan_bwd_saved")


def mamba_scan_fwd_noalloc(u, delta, delta_bias, A, B, C, D, z, y, last_state, *, stream=None):
    """The forward without any device allocation by the library: for callers
    that cannot let a library allocate (their own allocator owns device
    memory, or allocation calls are not allowed where they run).  Scratch lives
    in a fixed per-device array of the library; calls that overlap on the GPU
    race on it.  Same tensors as ``mamba_scan_fwd``."""
    batch, dim, L = u.shape
    N = A.shape[1]
    dt = u.dtype
    f32 = torch.float32
    args = [
        _ptr(u, dt, (batch, dim, L), "u"), _ptr(delta, dt, (batch, dim, L), "delta"),
        _ptr(delta_bias, f32, (dim,), "delta_bias"), _ptr(A, f32, (dim, N), "A"),
        _ptr(B, dt, (batch, N, L), "B"), _ptr(C, dt, (batch, N, L), "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, (batch, dim, L), "z"),
        _ptr(y, dt, (batch, dim, L), "y"), _ptr(last_state, f32, (batch, dim, N), "last_state"),
        batch, dim, L, N, _dtype_code(dt)]
    _check(load_library().mamba_scan_fwd_noalloc(*args, _stream_handle(stream)),
           "mamba_scan_fwd_noalloc")


def mamba_scan_step(state, u, delta, delta_bias, A, B, C, D, z, y, *, stream=None):
    """One decoding step (one token per batch row): updates ``state``
    (batch, dim, N) float32 in place and writes ``y`` (batch, dim).  u, delta,
    z, y: (batch, dim); B, C: (batch, N), in the I/O dtype."""
    batch, dim = u.shape
    N = A.shape[1]
    dt = u.dtype
    f32 = torch.float32
    args = [
        _ptr(state, f32, (batch, dim, N), "state"), _ptr(u, dt, (batch, dim), "u"),
        _ptr(delta, dt, (batch, dim), "delta"), _ptr(delta_bias, f32, (dim,), "delta_bias"),
        _ptr(A, f32, (dim, N), "A"), _ptr(B, dt, (batch, N), "B"), _ptr(C, dt, (batch, N), "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, (batch, dim), "z"), _ptr(y, dt, (batch, dim), "y"),
        batch, dim, N, _dtype_code(dt)]
    _check(load_library().mamba_scan_step(*args, _stream_handle(stream)), "mamba_scan_step")


def mamba_conv_scan_step(state, conv_state, x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z,
                         y, *, stream=None):
    """One decoding step with the convolution prologue: updates ``state``
    (batch, dim, N) and ``conv_state`` (batch, dim, W - 1) float32 in place
    and writes ``y`` (batch, dim).  x, delta, z, y: (batch, dim); B, C:
    (batch, N); conv_w (dim, W), conv_b (dim,) or None."""
    batch, dim = x.shape
    N = A.shape[1]
    W = conv_w.shape[1]
    dt = x.dtype
    f32 = torch.float32
    args = [
        _ptr(state, f32, (batch, dim, N), "state"),
        _ptr(conv_state, f32, (batch, dim, W - 1), "conv_state"), _ptr(x, dt, (batch, dim), "x"),
        _ptr(conv_w, f32, (dim, W), "conv_w"), _ptr(conv_b, f32, (dim,), "conv_b"), W,
        _ptr(delta, dt, (batch, dim), "delta"), _ptr(delta_bias, f32, (dim,), "delta_bias"),
        _ptr(A, f32, (dim, N), "A"), _ptr(B, dt, (batch, N), "B"), _ptr(C, dt, (batch, N), "C"),
        _ptr(D, f32, (dim,), "D"), _ptr(z, dt, (batch, dim), "z"), _ptr(y, dt, (batch, dim), "y"),
        batch, dim, N, _dtype_code(dt)]
    _check(load_library().mamba_conv_scan_step(*args, _stream_handle(stream)),
           "mamba_conv_scan_step")


class StepPlan:
    """A decoding plan (``mamba_scan_step_plan_create``): the buffers of one
    decoding token checked once; ``run()`` enqueues the step with a single
    kernel launch.  Write each token's u (or x), delta, z, B and C into the
    given tensors before its run.  With ``conv_w`` the plan steps the
    convolution prologue too (``conv_state`` (batch, dim, W - 1) float32,
    ``conv_b`` optional)."""

    def __init__(self, state, u, delta, delta_bias, A, B, C, D, z, y, *, conv_state=None,
                 conv_w=None, conv_b=None):
        batch, dim = u.shape
        N = A.shape[1]
        dt = u.dtype
        f32 = torch.float32
        W = conv_w.shape[1] if conv_w is not None else 0
        self._keep = (state, u, delta, delta_bias, A, B, C, D, z, y, conv_state, conv_w, conv_b)
        self._lib = load_library()
        self._h = ctypes.c_void_p()
        rc = self._lib.mamba_scan_step_plan_create(
            ctypes.byref(self._h), _ptr(state, f32, (batch, dim, N), "state"),
            _ptr(conv_state, f32, (batch, dim, max(W - 1, 0)), "conv_state") if W > 1 else None,
            _ptr(u, dt, (batch, dim), "u"),
            _ptr(conv_w, f32, (dim, W), "conv_w") if W else None,
            _ptr(conv_b, f32, (dim,), "conv_b") if W else None, W,
            _ptr(delta, dt, (batch, dim), "delta"), _ptr(delta_bias, f32, (dim,), "delta_bias"),
            _ptr(A, f32, (dim, N), "A"), _ptr(B, dt, (batch, N), "B"),
            _ptr(C, dt, (batch, N), "C"), _ptr(D, f32, (dim,), "D"),
            _ptr(z, dt, (batch, dim), "z"), _ptr(y, dt, (batch, dim), "y"),
            batch, dim, N, _dtype_code(dt))
        _check(rc, "mamba_scan_step_plan_create")
        # what run() needs, looked up once: the entry point, the handle as an
        # integer, the plan's device and torch's raw-stream query
        self._run = self._lib.mamba_scan_step_plan_run
        self._hv = self._h.value
        self._dev = u.device.index if u.device.index is not None else torch.cuda.current_device()
        self._raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)

    def run(self, stream=None):
        if stream is None and self._raw is not None:
            s = self._raw(self._dev)  # torch's current stream on the plan's device
        else:
            s = _stream_handle(stream)
        rc = self._run(self._hv, s)
        if rc:
            _check(rc, "mamba_scan_step_plan_run")

    def close(self):
        if self._h:
            self._lib.mamba_scan_step_plan_destroy(self._h)
            self._h = ctypes.c_void_p()
            self._hv = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def pool_set_reserve(nbytes: int) -> None:
    """Memory the library's workspace pool of the current device keeps mapped
    between calls (default 4 GiB)."""
    _check(load_library().mamba_scan_pool_set_reserve(int(nbytes)), "mamba_scan_pool_set_reserve")


def pool_trim(keep_bytes: int = 0) -> None:
    """Give the pool's unused memory on the current device back, down to
    ``keep_bytes``."""
    _check(load_library().mamba_scan_pool_trim(int(keep_bytes)), "mamba_scan_pool_trim")


def pool_reserved() -> int:
    """Bytes the library's workspace pool of the current device holds."""
    v = ctypes.c_uint64()
    _check(load_library().mamba_scan_pool_reserved(ctypes.byref(v)), "mamba_scan_pool_reserved")
    return int(v.value)


def test_fail_alloc(after: int) -> None:
    """Test hook: the workspace allocation after ``after`` more successful
    ones (on this thread) fails; negative disarms."""
    load_library().mamba_scan_test_fail_alloc(int(after))


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(load_library().mamba_scan_launch_count())


def mamba_scan_stream_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the sticky device status."""
    return load_library().mamba_scan_stream_status(_stream_handle(stream))


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                       return_last_state=False, path="auto", chunk_len=0, carry="auto",
                       stream=None):
    """Allocate y (and last_state) and run the forward; returns y or (y, last_state)."""
    batch, dim, L = u.shape
    y = torch.empty_like(u)
    last = (torch.empty(batch, dim, A.shape[1], device=u.device, dtype=torch.float32)
            if return_last_state else None)
    mamba_scan_fwd(u, delta, delta_bias, A, B, C, D, z, y, last, path=path,
                   chunk_len=chunk_len, carry=carry, stream=stream)
    return (y, last) if return_last_state else y


def selective_scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, path="auto",
                       chunk_len=0, carry="auto", stream=None) -> dict:
    """Allocate the gradients and run the backward; returns a dict of them."""
    dim, N = A.shape
    f32 = torch.float32
    g = {
        "du": torch.empty_like(u), "ddelta": torch.empty_like(u),
        "dA": torch.empty(dim, N, device=u.device, dtype=f32),
        "dB": torch.empty_like(B), "dC": torch.empty_like(C),
        "dD": torch.empty(dim, device=u.device, dtype=f32) if D is not None else None,
        "dz": torch.empty_like(u) if z is not None else None,
        "ddelta_bias": torch.empty(dim, device=u.device, dtype=f32),
    }
    mamba_scan_bwd(u, delta, delta_bias, A, B, C, D, z, dy, g["du"], g["ddelta"], g["dA"],
                   g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"], path=path,
                   chunk_len=chunk_len, carry=carry, stream=stream)
    return {k: v for k, v in g.items() if v is not None}


def selective_scan_fwd_save(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                            return_last_state=False, path="auto", chunk_len=0, carry="auto",
                            stream=None):
    """The forward of the training pair: allocates y (and last_state) and the
    saved buffer, runs ``mamba_scan_fwd_save``; returns (y, saved) or
    (y, last_state, saved).  ``saved`` is None where the problem saves
    nothing (``saved_bytes`` 0)."""
    batch, dim, L = u.shape
    N = A.shape[1]
    y = torch.empty_like(u)
    last = (torch.empty(batch, dim, N, device=u.device, dtype=torch.float32)
            if return_last_state else None)
    need = saved_bytes(batch, dim, L, N, u.dtype, path=path, chunk_len=chunk_len, carry=carry)
    saved = torch.empty(need, device=u.device, dtype=torch.uint8) if need else None
    mamba_scan_fwd_save(u, delta, delta_bias, A, B, C, D, z, y, last, saved, path=path,
                        chunk_len=chunk_len, carry=carry, stream=stream)
    return (y, last, saved) if return_last_state else (y, saved)


def selective_scan_bwd_saved(u, delta, A, B, C, dy, saved, D=None, z=None, delta_bias=None,
                             path="auto", chunk_len=0, carry="auto", stream=None) -> dict:
    """The backward of the training pair (``saved`` from
    ``selective_scan_fwd_save`` with the same inputs and options); returns
    the gradients as ``selective_scan_bwd`` does."""
    dim, N = A.shape
    f32 = torch.float32
    g = {
        "du": torch.empty_like(u), "ddelta": torch.empty_like(u),
        "dA": torch.empty(dim, N, device=u.device, dtype=f32),
        "dB": torch.empty_like(B), "dC": torch.empty_like(C),
        "dD": torch.empty(dim, device=u.device, dtype=f32) if D is not None else None,
        "dz": torch.empty_like(u) if z is not None else None,
        "ddelta_bias": torch.empty(dim, device=u.device, dtype=f32),
    }
    mamba_scan_bwd_saved(u, delta, delta_bias, A, B, C, D, z, dy, g["du"], g["ddelta"], g["dA"],
                         g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"], saved, path=path,
                         chunk_len=chunk_len, carry=carry, stream=stream)
    return {k: v for k, v in g.items() if v is not None}


def conv_selective_scan_fwd(x, conv_w, conv_b, delta, A, B, C, D=None, z=None, delta_bias=None,
                            return_last_state=False, path="auto", chunk_len=0, carry="auto",
                            stream=None):
    """Allocate y (and last_state) and run the forward with the convolution
    prologue; returns y or (y, last_state)."""
    batch, dim, L = x.shape
    y = torch.empty_like(x)
    last = (torch.empty(batch, dim, A.shape[1], device=x.device, dtype=torch.float32)
            if return_last_state else None)
    mamba_conv_scan_fwd(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, y, last, path=path,
                        chunk_len=chunk_len, carry=carry, stream=stream)
    return (y, last) if return_last_state else y


def conv_selective_scan_fwd_save(x, conv_w, conv_b, delta, A, B, C, D=None, z=None,
                                 delta_bias=None, return_last_state=False, path="auto",
                                 chunk_len=0, carry="auto", stream=None):
    """The training pair's forward with the convolution prologue; returns
    (y, saved) or (y, last_state, saved) as ``selective_scan_fwd_save``."""
    batch, dim, L = x.shape
    N = A.shape[1]
    y = torch.empty_like(x)
    last = (torch.empty(batch, dim, N, device=x.device, dtype=torch.float32)
            if return_last_state else None)
    need = conv_saved_bytes(batch, dim, L, N, conv_w.shape[1], x.dtype, path=path,
                            chunk_len=chunk_len, carry=carry)
    saved = torch.empty(need, device=x.device, dtype=torch.uint8) if need else None
    mamba_conv_scan_fwd_save(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, y, last, saved,
                             path=path, chunk_len=chunk_len, carry=carry, stream=stream)
    return (y, last, saved) if return_last_state else (y, saved)


def conv_selective_scan_bwd_saved(x, conv_w, conv_b, delta, A, B, C, dy, saved, D=None, z=None,
                                  delta_bias=None, path="auto", chunk_len=0, carry="auto",
                                  stream=None) -> dict:
    """The training pair's backward with the convolution prologue; returns
    the gradients as ``conv_selective_scan_bwd``."""
    dim, N = A.shape
    f32 = torch.float32
    g = {
        "dx": torch.empty_like(x), "dconv_w": torch.empty_like(conv_w),
        "dconv_b": torch.empty(dim, device=x.device, dtype=f32) if conv_b is not None else None,
        "ddelta": torch.empty_like(x),
        "dA": torch.empty(dim, N, device=x.device, dtype=f32),
        "dB": torch.empty_like(B), "dC": torch.empty_like(C),
        "dD": torch.empty(dim, device=x.device, dtype=f32) if D is not None else None,
        "dz": torch.empty_like(x) if z is not None else None,
        "ddelta_bias": torch.empty(dim, device=x.device, dtype=f32),
    }
    mamba_conv_scan_bwd_saved(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, dy, g["dx"],
                              g["dconv_w"], g["dconv_b"], g["ddelta"], g["dA"], g["dB"], g["dC"],
                              g["dD"], g["dz"], g["ddelta_bias"], saved, path=path,
                              chunk_len=chunk_len, carry=carry, stream=stream)
    return {k: v for k, v in g.items() if v is not None}


def conv_selective_scan_bwd(x, conv_w, conv_b, delta, A, B, C, dy, D=None, z=None,
                            delta_bias=None, path="auto", chunk_len=0, carry="auto",
                            stream=None) -> dict:
    """Allocate the gradients and run the backward with the convolution
    prologue; returns a dict of them (dx, dconv_w, dconv_b if conv_b is given,
    and the scan's other gradients)."""
    dim, N = A.shape
    f32 = torch.float32
    g = {
        "dx": torch.empty_like(x), "dconv_w": torch.empty_like(conv_w),
        "dconv_b": torch.empty(dim, device=x.device, dtype=f32) if conv_b is not None else None,
        "ddelta": torch.empty_like(x),
        "dA": torch.empty(dim, N, device=x.device, dtype=f32),
        "dB": torch.empty_like(B), "dC": torch.empty_like(C),
        "dD": torch.empty(dim, device=x.device, dtype=f32) if D is not None else None,
        "dz": torch.empty_like(x) if z is not None else None,
        "ddelta_bias": torch.empty(dim, device=x.device, dtype=f32),
    }
    mamba_conv_scan_bwd(x, conv_w, conv_b, delta, delta_bias, A, B, C, D, z, dy, g["dx"],
                        g["dconv_w"], g["dconv_b"], g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"],
                        g["dz"], g["ddelta_bias"], path=path, chunk_len=chunk_len, carry=carry,
                        stream=stream)
    return {k: v for k, v in g.items() if v is not None}
