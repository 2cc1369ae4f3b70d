"""Decode step on the GPU against the oracle's step, through the C ABI."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close
from structured_state_space_ssd_b200.inputs import make_inputs
from structured_state_space_ssd_b200.ssd import ssd_fwd, ssd_step

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "four_token_example.json")


def _token(inp, t, dev):
    """Token t of a make_inputs sequence, in the step's layouts."""
    return (inp["x"][:, t].contiguous().to(dev), inp["dt"][:, t].contiguous().to(dev), inp["A"].to(dev),
            inp["B"][:, t].contiguous().to(dev), inp["C"][:, t].contiguous().to(dev), inp["D"].to(dev))


STEP_CASES = [
    # batch, H, P, N, G, dtype
    (1, 2, 16, 16, 1, "f32"),
    (2, 6, 64, 128, 3, "f32"),
    (3, 4, 5, 7, 2, "f32"),      # N not a multiple of 4: one value per lane
    (2, 8, 64, 128, 1, "bf16"),
    (1, 3, 1, 1, 1, "bf16"),     # P = N = 1
    (1, 2, 64, 1024, 1, "f32"),  # largest N
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: "b{}_H{}_P{}_N{}_G{}_{}".format(*c))
def test_step_matches_oracle(case, cuda_device):
    b, H, P, N, G, dtype = case
    inp = make_inputs(b, 3, H, P, N, G, dtype, seed=11, with_init=True)
    state = inp["init_state"].clone()
    ref_state = state.double().numpy()
    st = state.to(cuda_device)
    for t in range(3):
        x, dt, A, B, C, D = _token(inp, t, cuda_device)
        y = ssd_step(st, x, dt, A, B, C, D)
        ref_state, y_ref = oracle.ssd_ref_step(ref_state, inp["x"][:, t], inp["dt"][:, t], inp["A"],
                                               inp["B"][:, t], inp["C"][:, t], inp["D"])
        torch.cuda.synchronize(cuda_device)
        assert_close(y.float().cpu().numpy(), y_ref, dtype, f"y, step {t}")
        assert_close(st.cpu().numpy(), ref_state, "f32", f"state, step {t}")


def test_four_token_example_on_the_gpu(cuda_device):
    with open(GOLDEN) as f:
        g = json.load(f)
    inp = g["inputs"]
    dev = cuda_device
    state = torch.zeros((1, 1, 1, 2), dtype=torch.float32, device=dev)
    A = torch.tensor([-1.0], device=dev)
    D = torch.tensor([0.0], device=dev)
    ys = []
    for t in range(4):
        x = torch.tensor([[[inp["x"][t]]]], dtype=torch.float32, device=dev)
        dt = torch.tensor([[-np.log(inp["a"][t])]], dtype=torch.float32, device=dev)
        B = torch.tensor([[inp["B"][t]]], dtype=torch.float32, device=dev)
        C = torch.tensor([[inp["C"][t]]], dtype=torch.float32, device=dev)
        ys.append(float(ssd_step(state, x, dt, A, B, C, D).item()))
    np.testing.assert_allclose(ys, g["printed"]["y_recurrence"], rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(state.cpu().numpy().reshape(2), g["derived_by_hand"]["final_state"],
                               rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_chained_steps_match_the_chunked_forward(dtype, cuda_device):
    # T decode steps from init_state give the y and final_state of one ssd_fwd over the T tokens
    b, T, H, P, N, G = 2, 40, 4, 64, 128, 2
    inp = make_inputs(b, T, H, P, N, G, dtype, seed=17, with_init=True)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    y_fwd, fin_fwd = ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 16, d["init_state"])
    st = d["init_state"].clone()
    ys = []
    for t in range(T):
        x, dt, A, B, C, D = _token(inp, t, cuda_device)
        ys.append(ssd_step(st, x, dt, A, B, C, D))
    y_step = torch.stack(ys, dim=1)
    torch.cuda.synchronize(cuda_device)
    assert_close(y_step.float().cpu().numpy(), y_fwd.float().cpu().numpy(), dtype, "y")
    assert_close(st.cpu().numpy(), fin_fwd.cpu().numpy(), "f32" if dtype == "f32" else dtype, "final_state")
