"""Parity report: the measured error of the CUDA path against the fp64 oracle
on every workload, per output tensor, at full size in the launch
configuration the benchmark times (auto path).

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
    y, last = gc.gpu_fwd(x)
    g = gc.gpu_bwd(x) if backward else None
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
    return 0


if __name__ == "__main__":
    sys.exit(main())
