"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the fp64 oracle on the same seeded inputs, and compare them normwise."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from selective_state_space_21_b200 import scan

# Tolerances on the normwise max error max|x - r| / max|r| per tensor.
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def normwise(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = max(float(np.abs(ref).max(initial=0.0)), 1e-300)
    return float(np.abs(got - ref).max(initial=0.0) / scale)


def to_device(x: dict, device="cuda") -> dict:
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in x.items()}


def to_host(x: dict) -> dict:
    return {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in x.items()}


def gpu_fwd(x: dict, path="auto", chunk_len=0, last=True, carry="auto"):
    out = scan.selective_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"],
                                  z=x["z"], delta_bias=x["delta_bias"],
                                  return_last_state=last, path=path, chunk_len=chunk_len,
                                  carry=carry)
    assert scan.mamba_scan_stream_status() == 0
    return out if last else (out, None)


def gpu_bwd(x: dict, path="auto", chunk_len=0, carry="auto") -> dict:
    g = scan.selective_scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"], D=x["D"],
                                z=x["z"], delta_bias=x["delta_bias"], path=path,
                                chunk_len=chunk_len, carry=carry)
    assert scan.mamba_scan_stream_status() == 0
    return g


def oracle_fwd(x: dict):
    return oracle.s6_forward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["delta_bias"],
                             x["D"], x["z"])


def oracle_bwd(x: dict) -> dict:
    return oracle.s6_backward(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"],
                              x["delta_bias"], x["D"], x["z"])


def sample_channels(batch: int, dim: int, k: int, seed: int = 0) -> dict:
    """k (batch, channel) pairs, spread over the grid (first and last channel
    of the first and last batch row included), grouped by batch row."""
    g = torch.Generator().manual_seed(seed)
    picks = {(0, 0), (batch - 1, dim - 1), (0, dim - 1), (batch - 1, 0)}
    while len(picks) < min(k, batch * dim):
        i = int(torch.randint(batch * dim, (1,), generator=g))
        picks.add((i // dim, i % dim))
    by_b: dict = {}
    for b, d in sorted(picks):
        by_b.setdefault(b, []).append(d)
    return by_b


def sample_channels_per_group(batch: int, dim: int, per_group: int, seed: int = 0,
                              group: int = 128) -> dict:
    """``per_group`` channels of every channel group of ``group`` channels in
    every batch row (the first and last channel of each group included, the
    rest drawn from a seeded generator), grouped by batch row."""
    g = torch.Generator().manual_seed(seed)
    by_b: dict = {}
    for b in range(batch):
        picks = set()
        for g0 in range(0, dim, group):
            g1 = min(dim, g0 + group)
            chosen = {g0, g1 - 1}
            while len(chosen) < min(per_group, g1 - g0):
                chosen.add(g0 + int(torch.randint(g1 - g0, (1,), generator=g)))
            picks |= chosen
        by_b[b] = sorted(picks)
    return by_b


def sub_problem(x: dict, b: int, ds: list) -> dict:
    """The inputs of batch row b restricted to channels ds (channels are
    independent, so the oracle can run on this slice alone)."""
    idx = torch.tensor(ds)
    pick = lambda t: None if t is None else t[b:b + 1].index_select(1, idx).contiguous()
    per_d = lambda t: None if t is None else t.index_select(0, idx).contiguous()
    return {
        "u": pick(x["u"]), "delta": pick(x["delta"]), "z": pick(x["z"]),
        "dy": pick(x.get("dy")), "B": x["B"][b:b + 1].contiguous(),
        "C": x["C"][b:b + 1].contiguous(), "A": per_d(x["A"]), "D": per_d(x["D"]),
        "delta_bias": per_d(x["delta_bias"]),
    }


def check_fwd_sampled(x_dev: dict, y: torch.Tensor, last: torch.Tensor, k: int, seed=0,
                      samples: dict = None):
    """Compare sampled channels of a full-size GPU forward with the oracle
    (``k`` channels from ``sample_channels``, or the given ``samples``).
    Returns the worst normwise errors of y and last_state."""
    batch, dim, _ = x_dev["u"].shape
    x = to_host(x_dev)
    y_h, last_h = y.cpu(), last.cpu() if last is not None else None
    ey = el = 0.0
    if samples is None:
        samples = sample_channels(batch, dim, k, seed)
    for b, ds in samples.items():
        sub = sub_problem(x, b, ds)
        y_ref, last_ref = oracle_fwd(sub)
        idx = torch.tensor(ds)
        ey = max(ey, normwise(y_h[b].index_select(0, idx).double().numpy(), y_ref[0]))
        if last_h is not None:
            el = max(el, normwise(last_h[b].index_select(0, idx).double().numpy(), last_ref[0]))
    return ey, el
