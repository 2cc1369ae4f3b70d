"""The forward with the block's gate and per-head GroupNorm (ssd_fwd_gated) against the oracle.

The reference is the oracle's forward followed by its gate + GroupNorm with one group per head, both
in fp64.  On the fused tensor-core path (P = 64, N <= 128) the gate runs in the kernel's drain on the
fp32 y; elsewhere ssd_fwd and ssd_gate_norm run one after the other.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close
from structured_state_space_ssd_b200 import make_inputs
from structured_state_space_ssd_b200 import ssd as S

pytestmark = pytest.mark.gpu

CASES = [
    # batch, T, H, P, N, G, Q, dtype, init, affine
    (2, 333, 4, 64, 128, 2, 256, "bf16", True, True),     # fused: ragged, grouped heads
    (1, 700, 6, 64, 64, 3, 128, "bf16", False, False),    # fused: one row block per chunk
    (1, 256, 2, 64, 16, 1, 256, "bf16", True, True),      # fused: small N, a single chunk
    (1, 8448, 2, 64, 128, 1, 256, "bf16", True, True),    # fused with the look-back chain (33 chunks)
    (1, 300, 2, 32, 64, 1, 256, "bf16", True, True),      # P = 32: forward, then the gate kernel
    (1, 300, 2, 64, 256, 2, 256, "bf16", False, True),    # N = 256: two launches, then the gate kernel
    (2, 100, 3, 16, 16, 1, 64, "f32", True, True),        # CUDA-core path, then the gate kernel
]


def _gated(case, dev):
    batch, T, H, P, N, G, Q, dtype, init, affine = case
    inp = make_inputs(batch, T, H, P, N, G, dtype, seed=900 + T + P, with_init=init)
    gen = torch.Generator().manual_seed(T * 7 + H)
    z = torch.randn(inp["x"].shape, generator=gen).to(inp["x"].dtype)
    w = (torch.rand(H * P, generator=gen) + 0.5) if affine else None
    b = torch.randn(H * P, generator=gen) if affine else None
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    out, fin = S.ssd_fwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], Q, z.to(dev), d["init_state"],
                               None if w is None else w.to(dev), None if b is None else b.to(dev), 1e-5)
    torch.cuda.synchronize(dev)
    y_ref, fin_ref = oracle.ssd_ref_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                        init_state=inp["init_state"])
    ref = oracle.ref_gate_norm(y_ref.reshape(batch * T, H * P), z.reshape(batch * T, H * P), H, 1e-5, w, b)
    return out, fin, ref.reshape(batch, T, H, P), fin_ref


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_T{}_H{}_P{}_N{}_G{}_Q{}_{}_{}_{}".format(*c))
def test_gated_forward_matches_oracle(case, cuda_device):
    out, fin, ref, fin_ref = _gated(case, cuda_device)
    dtype = case[7]
    assert_close(out.float().cpu().numpy(), ref, dtype, "gated output")
    assert_close(fin.cpu().numpy(), fin_ref, dtype, "final_state")


def test_gated_launch_counts(cuda_device):
    lib = S.load()
    assert lib.ssd_fwd_gated_launch_count(4, 2048, 80, 64, 1, 128, 256, S.SSD_BF16) == 1   # in the drain
    assert lib.ssd_fwd_gated_launch_count(1, 300, 2, 32, 1, 64, 256, S.SSD_BF16) == 2     # + gate kernel
    assert lib.ssd_fwd_gated_launch_count(1, 300, 2, 64, 2, 256, 256, S.SSD_BF16) == 3    # 2 + gate kernel
    assert lib.ssd_fwd_gated_launch_count(1, 100, 3, 16, 1, 16, 64, S.SSD_F32) == 5       # 4 + gate kernel


def test_gated_forward_is_deterministic_and_matches_the_two_step_path(cuda_device):
    # fused drain vs ssd_fwd + ssd_gate_norm on the same inputs: equal up to the bf16 rounding of y
    case = (2, 600, 8, 64, 128, 1, 256, "bf16", True, True)
    out1, _, ref, _ = _gated(case, cuda_device)
    out2, _, _, _ = _gated(case, cuda_device)
    assert torch.equal(out1, out2)
    batch, T, H, P, N, G, Q = case[:7]
    inp = make_inputs(batch, T, H, P, N, G, "bf16", seed=900 + T + P, with_init=True)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    gen = torch.Generator().manual_seed(T * 7 + H)
    z = torch.randn(inp["x"].shape, generator=gen).to(torch.bfloat16)
    w = torch.rand(H * P, generator=gen) + 0.5
    b = torch.randn(H * P, generator=gen)
    y, _ = S.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], Q, d["init_state"])
    two = S.ssd_gate_norm(y.view(batch * T, H * P), z.to(cuda_device).view(batch * T, H * P), H, 1e-5,
                          w.to(cuda_device), b.to(cuda_device))
    torch.cuda.synchronize(cuda_device)
    assert_close(two.float().cpu().numpy().reshape(ref.shape), ref, "bf16", "two-step path")
    diff = (two.float().view(out1.shape) - out1.float()).abs().max().item()
    assert diff < 0.1, diff


def test_gated_forward_rejects_bad_arguments(cuda_device):
    inp = make_inputs(1, 128, 2, 64, 64, 1, "bf16", seed=5)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    z = torch.zeros_like(d["x"])
    with pytest.raises(ValueError):
        S.ssd_fwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256, z.float())      # z dtype
    with pytest.raises(ValueError):
        S.ssd_fwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256, z,
                        norm_weight=torch.ones(5, device=cuda_device))                         # weight size
    with pytest.raises(S.SSDError):
        S.ssd_fwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256, z, eps=-1.0)    # eps < 0
    with pytest.raises(S.SSDError):
        S.ssd_fwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256, z, out=z)       # out is z
