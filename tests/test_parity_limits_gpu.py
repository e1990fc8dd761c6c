"""GPU parity at the limits of the step size Delta, against the fp64 oracle.

The two regimes the pages single out ("Mamba: Linear-Time Sequence Modeling
with Selective State Spaces", chapterpal.com, Knowl 4; the paper-graph-ui
summary, section 3.5 "Theoretical Connections: Selection as Generalized
Gating"): a large Delta resets the state to the current input (for a
diagonal A the memoryless state h = -B u / A), a small Delta keeps it.
Delta = softplus(delta + bias), so a bias of +-30 / +-60 / +-90 drives
every step of every channel into a limit.  The cases run each arithmetic of
the kernels (A = -(n+1) with the sigmoid identity, scaled S4D-Real A, an
unstructured A), the staged kernels with and without the structured
arithmetic and the one-thread-per-channel kernels, forward and backward,
plus mixtures of the limits inside one channel group and inside one
sequence, and token-by-token decoding.
"""
import numpy as np
import pytest
import torch

import gpu_cases as gc
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

MODES = ["sig", "struct", "generic"]
PATHS = ["auto", "generic", "reference"]
GRADS = ["du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()


def limit_inputs(regime, mode, dtype, b=2, d=160, L=512, N=16, seed=7):
    """Workload-shaped inputs whose Delta sits in a limit.  `regime`: 'large<v>'
    / 'small<v>' set every channel's bias to +v / -v; 'mix' cycles the
    channels of each group through +30, -30, +60, -60 and the drawn bias;
    'held' / 'reset' shift delta by -60 / +60 over the second half of every
    sequence.  `mode` picks A: 'sig' is -(n+1); 'struct' is -(n+1) times a
    per-channel scale; 'generic' is -exp(N(0, 1)) per state."""
    x = make_inputs(b, d, L, N, dtype, seed=seed, with_dy=True)
    g = torch.Generator().manual_seed(seed + 1)
    if mode == "struct":
        s = torch.exp(torch.randn(d, 1, generator=g) * 0.7)
        x["A"] = (-torch.arange(1, N + 1, dtype=torch.float32)[None, :] * s).contiguous()
    elif mode == "generic":
        x["A"] = (-torch.exp(torch.randn(d, N, generator=g))).contiguous()
    bias = x["delta_bias"].clone()
    if regime.startswith(("large", "small")):
        v = float(regime[5:]) * (1.0 if regime.startswith("large") else -1.0)
        bias = torch.full((d,), v)
    elif regime == "mix":
        vals = torch.tensor([30.0, -30.0, 60.0, -60.0, 0.0])
        sel = vals[torch.arange(d) % 5]
        bias = torch.where(sel == 0, bias, sel)
    elif regime in ("held", "reset"):
        dl = x["delta"].float()
        dl[:, :, L // 2:] += -60.0 if regime == "held" else 60.0
        x["delta"] = dl.to(dtype)
    x["delta_bias"] = bias.contiguous()
    return x
