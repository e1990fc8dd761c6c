"""Parity report: the measured error of the CUDA path against the fp64 oracle
on every workload, per output tensor, at full size in the launch
configuration the benchmark times (auto path; the training pair where the
workload has a backward), and of the convolution
prologue, the Delta projection and complex A on the bf16 2K workload.

    python tests/parity_report.py            # needs a B200; prints a markdown table

For each tensor it gives the normwise max error max|x - r| / max|r| (the bar:
1e-4 for fp32 I/O, 2e-2 for bf16 I/O) and the 99.9th percentile of the
elementwise error |x - r| / max(|r|, 1e-3 max|r|).  Channels are sampled
where the oracle would take too long on all of them; dB and dC, which sum
over every channel, are compared on one whole batch row.  Test
infrastructure: it runs the oracle."""
from __future__ import annotations

import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import gpu_cases as gc  # noqa: E402
from selective_state_space_21_b200 import build, scan  # noqa: E402
from selective_state_space_21_b200.inputs import WORKLOADS, workload_inputs  # noqa: E402


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = max(float(np.abs(ref).max(initial=0.0)), 1e-300)
    d = np.abs(got - ref)
    rel = d / np.maximum(np.abs(ref), 1e-3 * scale)
    return float(d.max(initial=0.0) / scale), float(np.percentile(rel, 99.9)) if rel.size else 0.0


def report(index: int, k: int, backward: bool):
    w = WORKLOADS[index]
    x = workload_inputs(index, device="cuda", with_dy=backward)
    if backward:  # the training pair, as the benchmark times it
        y, last, saved = scan.selective_scan_fwd_save(
            x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
            delta_bias=x["delta_bias"], return_last_state=True)
        g = scan.selective_scan_bwd_saved(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dy"],
                                          saved, D=x["D"], z=x["z"], delta_bias=x["delta_bias"])
        assert scan.mamba_scan_stream_status() == 0
    else:
        y, last = gc.gpu_fwd(x)
        g = None
    xh = gc.to_host(x)
    yh, lh = y.cpu(), last.cpu()
    gh = {key: v.cpu() for key, v in g.items()} if g else {}
    acc: dict = {}

    def add(name, got, ref):
        e = errors(got, ref)
        a = acc.setdefault(name, [0.0, 0.0])
        a[0], a[1] = max(a[0], e[0]), max(a[1], e[1])

    for b, ds in gc.sample_channels(w.batch, w.dim, k, seed=index).items():
        idx = torch.tensor(ds)
        sub = gc.sub_problem(xh, b, ds)
        y_ref, last_ref = gc.oracle_fwd(sub)
        add("y", yh[b].index_select(0, idx).double().numpy(), y_ref[0])
        add("last_state", lh[b].index_select(0, idx).double().numpy(), last_ref[0])
        if backward:
            ref = gc.oracle_bwd(sub)
            for key in ("du", "ddelta", "dz"):
                add(key, gh[key][b].index_select(0, idx).double().numpy(), ref[key][0])
    if backward:
        b = w.batch - 1
        ref = gc.oracle_bwd(gc.sub_problem(xh, b, list(range(w.dim))))
        for key in ("dB", "dC"):
            add(key, gh[key][b].double().numpy(), ref[key][0])
        ds = [0, w.dim // 2 + 1, w.dim - 1]
        idx = torch.tensor(ds)
        sub = {key: xh[key].index_select(1, idx).contiguous() for key in ("u", "delta", "z", "dy")}
        sub.update(B=xh["B"], C=xh["C"], A=xh["A"].index_select(0, idx).contiguous(),
                   D=xh["D"].index_select(0, idx).contiguous(),
                   delta_bias=xh["delta_bias"].index_select(0, idx).contiguous())
        ref = gc.oracle_bwd(sub)
        for key in ("dA", "dD", "ddelta_bias"):
            add(key, gh[key].index_select(0, idx).double().numpy(), ref[key])
    return w, acc


def report_variant(kind: str, k: int = 16):
    """The rows beyond the plain scan on the bf16 8 x 5120 x 2048 workload:
    the convolution prologue (width 4, through its training pair), the
    rank-160 Delta projection and
    complex A with 16 complex states.  y and the per-channel gradients on
    sampled channels; the per-channel parameters' gradients (summed over the
    batch) on three channels."""
    import test_parity_conv_gpu as tc
    import test_parity_cplx_gpu as tx
    import test_parity_dtproj_gpu as td
    from selective_state_space_21_b200.inputs import make_cplx_inputs

    w = WORKLOADS[2]
    if kind == "conv":
        xh = tc.conv_case(w.batch, w.dim, w.L, w.N, w.dtype, seed=1236)
        ofwd, obwd = tc.oracle_fwd, tc.oracle_bwd
        rows, per_d, grads, params = ("u", "delta", "z", "dy"), ("A", "D", "delta_bias", "conv_w",
                                      "conv_b"), ("dx", "ddelta", "dz"), ("dconv_w", "dconv_b", "dA")
    elif kind == "dtproj":
        xh = td.case(w.batch, w.dim, w.L, w.N, (w.dim // 2 + 15) // 16, w.dtype, seed=1194)
        ofwd, obwd = td.oracle_fwd, td.oracle_bwd
        rows, per_d, grads, params = ("u", "z", "dy"), ("A", "D", "delta_bias", "W_dt"), \
            ("du", "dz"), ("dW_dt", "dA")
    else:
        xh = make_cplx_inputs(w.batch, w.dim, w.L, w.N, w.dtype, seed=1396, with_dy=True)
        ofwd = lambda x: tx.oracle.s6_cplx_forward(x["u"], x["delta"], x["A"], x["B"], x["C"],
                                                   delta_bias=x["delta_bias"], D=x["D"], z=x["z"])
        obwd = lambda x: tx.oracle.s6_cplx_backward(x["u"], x["delta"], x["A"], x["B"], x["C"],
                                                    x["dy"], delta_bias=x["delta_bias"], D=x["D"],
                                                    z=x["z"])
        rows, per_d, grads, params = ("u", "delta", "z", "dy"), ("A", "D", "delta_bias"), \
            ("du", "ddelta", "dz"), ("dA", "dD", "ddelta_bias")
    x = gc.to_device(xh)
    if kind == "conv":  # the training pair, as the benchmark times it
        kw = dict(D=x["D"], z=x["z"], delta_bias=x["delta_bias"])
        yd, saved = scan.conv_selective_scan_fwd_save(x["u"], x["conv_w"], x["conv_b"], x["delta"],
                                                      x["A"], x["B"], x["C"], **kw)
        gd = scan.conv_selective_scan_bwd_saved(x["u"], x["conv_w"], x["conv_b"], x["delta"],
                                                x["A"], x["B"], x["C"], x["dy"], saved, **kw)
        assert scan.mamba_scan_stream_status() == 0
        y = yd.cpu()
        g = {key: v.cpu() for key, v in gd.items() if v is not None}
    else:  # the projection's and complex A's training pairs, also as the benchmark times them
        if kind == "dtproj":
            _, yd, _, gd = td.gpu_pair(x)
        else:
            yd, _, gd = tx.pair(x)
        y = yd.cpu()
        g = {key: v.cpu() for key, v in gd.items() if v is not None}
    acc: dict = {}

    def add(name, got, ref):
        e = errors(got, ref)
        a = acc.setdefault(name, [0.0, 0.0])
        a[0], a[1] = max(a[0], e[0]), max(a[1], e[1])

    def shared(b):  # tensors shared by the channels of batch row b
        out = {"B": xh["B"][b:b + 1].contiguous(), "C": xh["C"][b:b + 1].contiguous()}
        if "dt_low" in xh:
            out["dt_low"] = xh["dt_low"][b:b + 1].contiguous()
        return out

    for b, ds in gc.sample_channels(w.batch, w.dim, k, seed=5).items():
        idx = torch.tensor(ds)
        sub = {n: xh[n][b:b + 1].index_select(1, idx).contiguous() for n in rows}
        sub.update({n: xh[n].index_select(0, idx).contiguous() for n in per_d})
        sub.update(shared(b))
        if "delta" not in sub:
            sub["delta"] = None
        y_ref = ofwd(sub)[0]
        add("y", y[b].index_select(0, idx).double().numpy(), y_ref[0])
        ref = obwd(sub)
        for key in grads:
            add(key, g[key][b].index_select(0, idx).double().numpy(), ref[key][0])
    idx = torch.tensor([0, w.dim // 2 + 1, w.dim - 1])
    sub = {n: xh[n].index_select(1, idx).contiguous() for n in rows}
    sub.update({n: xh[n].index_select(0, idx).contiguous() for n in per_d})
    sub.update(B=xh["B"], C=xh["C"])
    if "dt_low" in xh:
        sub["dt_low"] = xh["dt_low"]
    ref = obwd(sub)
    for key in params:
        add(key, g[key].index_select(0, idx).double().numpy(), ref[key])
    return acc


def main():
    build.build()
    scan.load_library()
    cases = [(1, 48, True), (2, 48, True), (3, 12, False), (4, 48, True)]
    print("| workload | tensor | normwise max error | 99.9th pct elementwise | bar |")
    print("|---|---|---|---|---|")
    for index, k, backward in cases:
        w, acc = report(index, k, backward)
        bar = gc.TOL[w.dtype]
        for name, (e, p) in acc.items():
            print(f"| {w.name} | {name} | {e:.2e} | {p:.2e} | {bar:g} |", flush=True)
    names = {"conv": "convolution prologue (width 4)", "dtproj": "Δ projection (R = 160)",
             "cplx": "complex A (16 complex states)"}
    for kind in ("conv", "dtproj", "cplx"):
        for name, (e, p) in report_variant(kind).items():
            print(f"| {WORKLOADS[2].name}, {names[kind]} | {name} | {e:.2e} | {p:.2e} | 0.02 |",
                  flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
