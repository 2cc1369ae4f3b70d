"""Sequence split on one GPU: shards run from a zero state, exchange states, and correct their outputs.

The shards of one sequence are processed here one after another on one GPU
(the multi-worker exchange is the same all-gather that test_multirank runs on
gloo); the assembled output must be the forward over the whole sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close
from structured_state_space_ssd_b200.inputs import make_inputs
from structured_state_space_ssd_b200.ssd import (ssd_fwd, ssd_split_combine, ssd_split_correct,
                                                 ssd_split_logdecay)

pytestmark = pytest.mark.gpu


def _split_forward(d, cuts, Q):
    """Run the shards [cuts[k], cuts[k+1]) through steps 1-5 of the split; returns (y, final_state)."""
    parts = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sl = {k: d[k][:, a:b].contiguous() for k in ("x", "dt", "B", "C")}
        y0, fin0 = ssd_fwd(sl["x"], sl["dt"], d["A"], sl["B"], sl["C"], d["D"], Q, None)
        sig, total = ssd_split_logdecay(sl["dt"], d["A"])
        parts.append((y0, fin0, sig, total, sl["C"]))
    fin0_all = torch.stack([p[1] for p in parts])
    total_all = torch.stack([p[3] for p in parts])
    ys, fin = [], None
    for k, (y0, _, sig, _, Ck) in enumerate(parts):
        s_in, fin = ssd_split_combine(fin0_all, total_all, k, d["init_state"])
        ys.append(ssd_split_correct(y0, Ck, sig, s_in))
    return torch.cat(ys, dim=1), fin


CASES = [
    # batch, T, H, P, N, G, dtype, init, shard cuts
    (1, 300, 4, 16, 16, 2, "f32", True, [0, 300]),
    (2, 700, 6, 64, 128, 3, "f32", True, [0, 256, 512, 700]),
    (2, 1000, 8, 64, 128, 2, "bf16", True, [0, 100, 611, 1000]),
    (1, 2048, 4, 64, 64, 1, "bf16", False, [0, 512, 1024, 1536, 2048]),
    (1, 333, 2, 32, 256, 1, "f32", True, [0, 1, 200, 333]),   # a one-token shard
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_T{}_H{}_P{}_N{}_G{}_{}_{}_K{}".format(*c[:8], len(c[8]) - 1))
def test_split_matches_oracle(case, cuda_device):
    b, T, H, P, N, G, dtype, init, cuts = case
    inp = make_inputs(b, T, H, P, N, G, dtype, seed=41, with_init=init)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    y, fin = _split_forward(d, cuts, 128 if P <= 32 else 256)
    torch.cuda.synchronize(cuda_device)
    y_ref, fin_ref = oracle.ssd_ref_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                        init_state=inp["init_state"])
    assert_close(y.float().cpu().numpy(), y_ref, dtype, "y")
    assert_close(fin.cpu().numpy(), fin_ref, "f32" if dtype == "f32" else dtype, "final_state")


def test_logdecay_prefix_and_total(cuda_device):
    inp = make_inputs(2, 777, 5, 8, 8, 1, "f32", seed=3)
    sig, total = ssd_split_logdecay(inp["dt"].to(cuda_device), inp["A"].to(cuda_device))
    ref = np.cumsum(inp["dt"].double().numpy() * inp["A"].double().numpy()[None, None, :], axis=1)  # [b,T,H]
    np.testing.assert_allclose(sig.cpu().numpy(), ref.transpose(0, 2, 1), rtol=1e-5, atol=1e-4)
    np.testing.assert_allclose(total.cpu().numpy(), ref[:, -1, :], rtol=1e-5, atol=1e-4)
