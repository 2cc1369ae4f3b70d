"""Swish gate + GroupNorm on the GPU against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close
from structured_state_space_ssd_b200.ssd import ssd_gate_norm

pytestmark = pytest.mark.gpu

CASES = [
    # rows, channels, ngroups, dtype, affine
    (7, 64, 1, "f32", False),
    (33, 5120, 80, "bf16", True),    # the 2.7B layer's H * P with a group per head
    (5, 5120, 8, "bf16", False),     # groups of 640 channels
    (3, 96, 12, "bf16", True),       # groups of 8
    (4, 36, 3, "bf16", False),       # groups of 12: no 16-byte path
    (2, 4096, 1, "f32", True),       # the largest group
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "r{}_C{}_g{}_{}_{}".format(*c))
def test_gate_norm_matches_oracle(case, cuda_device):
    rows, ch, ng, dtype, affine = case
    g = torch.Generator().manual_seed(rows * 131 + ch)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    y = (torch.randn((rows, ch), generator=g) * 2.0).to(tdt)
    z = torch.randn((rows, ch), generator=g).to(tdt)
    w = torch.rand(ch, generator=g) + 0.5 if affine else None
    b = torch.randn(ch, generator=g) if affine else None
    dev = cuda_device
    out = ssd_gate_norm(y.to(dev), z.to(dev), ng, 1e-5, None if w is None else w.to(dev),
                        None if b is None else b.to(dev))
    torch.cuda.synchronize(dev)
    ref = oracle.ref_gate_norm(y, z, ng, 1e-5, w, b)
    assert_close(out.float().cpu().numpy(), ref, dtype, "gate_norm")


def test_gate_norm_in_place_on_the_layer_output(cuda_device):
    y = torch.randn((16, 320), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    z = torch.randn((16, 320), generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    ref = oracle.ref_gate_norm(y, z, 5)
    yd = y.to(cuda_device)
    out = ssd_gate_norm(yd, z.to(cuda_device), 5, out=yd)
    torch.cuda.synchronize(cuda_device)
    assert out.data_ptr() == yd.data_ptr()
    assert_close(yd.float().cpu().numpy(), ref, "bf16", "gate_norm in place")
