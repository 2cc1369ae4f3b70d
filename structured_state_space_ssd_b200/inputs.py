"""Seeded synthetic inputs for the SSD layer forward.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests, so it holds none of the layer's arithmetic: it only draws the inputs.

Value distributions (identical for every workload):

* ``x ~ N(0, 1)``; ``B, C ~ N(0, 1) / sqrt(N)``;
* ``dt = softplus(z + bias)`` with ``z ~ N(0, 1)`` and one fixed bias
  ``ln(e^0.01 - 1)`` (about -4.600), so that ``dt`` lies in [1e-3, 0.1] for
  about 98% of the draws.  ``dt`` arrives final: the layer applies no softplus,
  bias or clamp of its own;
* ``A_h = -exp(U(ln 1, ln 16))``; ``D ~ N(0, 1)``;
* ``init_state ~ N(0, 0.1^2)`` when the workload has one, else none (zero).

Everything is drawn in fp32 on the CPU with ``torch.Generator``; for bf16
workloads ``x``, ``B`` and ``C`` are then rounded once to bf16 (round to
nearest even) and both the CUDA path and the oracle consume those rounded
values.  ``dt``, ``A``, ``D`` and the states stay fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DT_BIAS = math.log(math.expm1(0.01))  # about -4.600


@dataclass(frozen=True)
class Workload:
    """One SSD forward problem: shapes, dtype, chunk size and seed."""
    name: str
    batch: int
    T: int
    H: int
    P: int
    N: int
    G: int
    Q: int
    dtype: str  # "f32" or "bf16": dtype of x, B, C and y
    seed: int
    with_init: bool = False
    note: str = field(default="", compare=False)

    @property
    def tokens(self) -> int:
        return self.batch * self.T

    @property
    def nc(self) -> int:
        return -(-self.T // self.Q)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_f32", 1, 256, 2, 16, 16, 1, 64, "f32", 1000,
                 note="batch 1, T=256, H=2, P=16, N=16, G=1, Q=64, fp32"),
        Workload("mamba2_130m_layer", 8, 2048, 24, 64, 128, 1, 256, "bf16", 1001,
                 note="batch 8, T=2048, d_inner 1536 -> H=24, P=64, N=128, G=1, Q=256, bf16"),
        Workload("mamba2_2p7b_layer", 4, 2048, 80, 64, 128, 1, 256, "bf16", 1002,
                 note="batch 4, T=2048, d_inner 5120 -> H=80, P=64, N=128, G=1, Q=256, bf16"),
        Workload("nsweep_N16", 8, 4096, 32, 64, 16, 1, 256, "bf16", 3016),
        Workload("nsweep_N64", 8, 4096, 32, 64, 64, 1, 256, "bf16", 3064),
        Workload("nsweep_N128", 8, 4096, 32, 64, 128, 1, 256, "bf16", 3128),
        Workload("nsweep_N256", 8, 4096, 32, 64, 256, 1, 256, "bf16", 3256),
        Workload("long_131k", 1, 131072, 48, 64, 128, 8, 256, "bf16", 1004, with_init=True,
                 note="batch 1, T=131072, H=48, P=64, N=128, G=8, Q=256, bf16, init ~ N(0, 0.1^2)"),
    ]
}

HEADLINE = "mamba2_2p7b_layer"


def make_inputs(batch: int, T: int, H: int, P: int, N: int, G: int, dtype: str = "bf16",
                seed: int = 0, with_init: bool = False, device: str = "cpu") -> dict:
    """Draw one problem's inputs (see the module docstring).

    Returns a dict of tensors: x [b,T,H,P], dt [b,T,H], A [H], B, C
    [b,T,G,N], D [H] and init_state [b,H,P,N] or None.  x/B/C have dtype
    ``torch.float32`` or ``torch.bfloat16``; the rest are fp32.  With the
    default ``device="cpu"`` the draws are reproducible across machines (every
    parity test uses them); another device draws the same distributions with
    that device's generator, for timing runs that need no oracle.
    """
    if dtype not in ("f32", "bf16"):
        raise ValueError(f"dtype must be 'f32' or 'bf16', got {dtype!r}")
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    kw = dict(generator=g, device=device)
    x = torch.randn(batch, T, H, P, **kw)
    B = torch.randn(batch, T, G, N, **kw) / math.sqrt(N)
    C = torch.randn(batch, T, G, N, **kw) / math.sqrt(N)
    dt = torch.nn.functional.softplus(torch.randn(batch, T, H, **kw) + DT_BIAS)
    A = -torch.exp(torch.empty(H, device=device).uniform_(math.log(1.0), math.log(16.0), generator=g))
    D = torch.randn(H, **kw)
    init = (0.1 * torch.randn(batch, H, P, N, **kw)) if with_init else None
    if dtype == "bf16":
        x, B, C = x.bfloat16(), B.bfloat16(), C.bfloat16()
    return {"x": x, "dt": dt, "A": A, "B": B, "C": C, "D": D, "init_state": init}


def workload_inputs(w: Workload) -> dict:
    """Inputs of a named workload, drawn with its own seed."""
    return make_inputs(w.batch, w.T, w.H, w.P, w.N, w.G, w.dtype, w.seed, w.with_init)


def make_output_grads(batch: int, T: int, H: int, P: int, N: int, dtype: str = "bf16", seed: int = 0,
                      with_dfinal: bool = False) -> dict:
    """Draw the gradients arriving at the layer's outputs for a backward pass.

    Returns CPU tensors ``dy`` [b,T,H,P] ~ N(0, 1) in the dtype of y (rounded once
    to bf16 for bf16 problems) and ``dfinal_state`` [b,H,P,N] ~ N(0, 0.1^2) in fp32,
    or None.  The seed stream is separate from :func:`make_inputs`'.
    """
    if dtype not in ("f32", "bf16"):
        raise ValueError(f"dtype must be 'f32' or 'bf16', got {dtype!r}")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7_000_003)
    dy = torch.randn(batch, T, H, P, generator=g)
    dfin = (0.1 * torch.randn(batch, H, P, N, generator=g)) if with_dfinal else None
    if dtype == "bf16":
        dy = dy.bfloat16()
    return {"dy": dy, "dfinal_state": dfin}
