"""Backward pass on the GPU against the fp64 backward oracle, through the C ABI.

Tolerances (max_rel = max|err| / max|ref| and rel_l2, per gradient tensor):

* gradients in the input dtype (dx, dB, dC): the forward's bars -- fp32 1e-4;
  bf16 2e-2 / 5e-3, the outputs being rounded once to bf16;
* fp32 gradients (ddt, dD, dinit_state), either input dtype: 1e-4, all of
  their arithmetic being fp32 (fp64 for the sums over the sequence) on exact
  inputs;
* dA: 1e-3.  dA_h is a sum over every (batch, token) whose absolute sum
  exceeds |dA_h| by factors up to about 90 on these inputs, so a 1e-5
  relative error of the fp32 terms shows as up to 1e-3 in the result.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, metrics
from structured_state_space_ssd_b200.inputs import WORKLOADS, make_inputs, make_output_grads, workload_inputs
from structured_state_space_ssd_b200.ssd import ssd_bwd, ssd_fwd, ssd_layer

pytestmark = pytest.mark.gpu

F32_TOL = {"max_rel": 1e-4, "rel_l2": 1e-4}
DA_TOL = {"max_rel": 1e-3, "rel_l2": 1e-3}
DTYPE_GRADS = ("dx", "dB", "dC")  # in the input dtype; every other gradient is fp32


def _check(name, got, ref, dtype):
    tol = TOL[dtype] if name in DTYPE_GRADS else (DA_TOL if name == "dA" else F32_TOL)
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{name}: non-finite"
    m = metrics(got, ref)
    assert m["max_rel"] <= tol["max_rel"] and m["rel_l2"] <= tol["rel_l2"], f"{name}: {m} vs {tol}"
    return m


def _to(dev, d):
    return {k: (None if v is None else v.to(dev)) for k, v in d.items()}


def _run(inp, grads, Q, dev):
    d, g = _to(dev, inp), _to(dev, grads)
    out = ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], g["dy"], Q, d["init_state"], g["dfinal_state"])
    torch.cuda.synchronize(dev)
    return {k: (None if v is None else v.float().cpu().numpy()) for k, v in out.items()}


CASES = [
    # batch, T, H, P, N, G, Q, dtype, init, dfinal
    (1, 256, 2, 16, 16, 1, 64, "f32", False, False),
    (2, 700, 4, 64, 128, 2, 256, "f32", True, True),        # ragged last chunk, groups
    (2, 700, 8, 64, 128, 1, 256, "bf16", True, True),
    (1, 300, 4, 128, 256, 4, 128, "f32", False, True),      # largest P and N
    (1, 129, 3, 32, 64, 3, 64, "bf16", True, False),        # one row past a chunk
    (3, 1, 2, 8, 8, 1, 16, "f32", True, True),              # a single token
    (1, 64, 6, 64, 128, 2, 256, "bf16", False, False),      # T < Q
    (2, 600, 4, 64, 64, 2, 128, "bf16", True, True),        # tensor-core scans at N = 64, Q = 128
    (1, 200, 2, 5, 7, 1, 32, "f32", True, True),            # odd P and N
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_T{}_H{}_P{}_N{}_G{}_Q{}_{}_{}{}".format(
    *c[:8], "i" if c[8] else "", "f" if c[9] else ""))
def test_backward_matches_oracle(case, cuda_device):
    b, T, H, P, N, G, Q, dtype, init, dfin = case
    inp = make_inputs(b, T, H, P, N, G, dtype, seed=41, with_init=init)
    grads = make_output_grads(b, T, H, P, N, dtype, seed=41, with_dfinal=dfin)
    got = _run(inp, grads, Q, cuda_device)
    ref = oracle.ssd_ref_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], grads["dy"],
                             init_state=inp["init_state"], dfinal_state=grads["dfinal_state"])
    for name in ("dx", "dB", "dC", "ddt", "dA", "dD", "dinit_state"):
        _check(name, got[name], ref[name], dtype)


def test_empty_sequence_passes_the_final_gradient_through(cuda_device):
    inp = make_inputs(2, 0, 3, 16, 32, 1, "f32", seed=42, with_init=True)
    grads = make_output_grads(2, 0, 3, 16, 32, "f32", seed=42, with_dfinal=True)
    got = _run(inp, grads, 64, cuda_device)
    np.testing.assert_array_equal(got["dinit_state"], grads["dfinal_state"].numpy())
    assert np.all(got["dA"] == 0) and np.all(got["dD"] == 0) and got["dx"].size == 0


def test_repeated_backward_is_bitwise_identical(cuda_device):
    inp = make_inputs(2, 1000, 8, 64, 128, 2, "bf16", seed=43, with_init=True)
    grads = make_output_grads(2, 1000, 8, 64, 128, "bf16", seed=43, with_dfinal=True)
    first = _run(inp, grads, 256, cuda_device)
    for _ in range(2):
        again = _run(inp, grads, 256, cuda_device)
        for k, v in first.items():
            assert np.array_equal(v, again[k]), k


def test_autograd_layer_gives_the_library_gradients(cuda_device):
    inp = make_inputs(1, 300, 4, 64, 128, 2, "bf16", seed=44, with_init=True)
    grads = make_output_grads(1, 300, 4, 64, 128, "bf16", seed=44, with_dfinal=True)
    d, g = _to(cuda_device, inp), _to(cuda_device, grads)
    leaves = {k: d[k].clone().requires_grad_(True) for k in ("x", "dt", "A", "B", "C", "D", "init_state")}
    y, fin = ssd_layer(leaves["x"], leaves["dt"], leaves["A"], leaves["B"], leaves["C"], leaves["D"], 256,
                       leaves["init_state"])
    y_ref, fin_ref = ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256, d["init_state"])
    assert torch.equal(y, y_ref) and torch.equal(fin, fin_ref)
    torch.autograd.backward((y, fin), (g["dy"], g["dfinal_state"]))
    direct = ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], g["dy"], 256, d["init_state"],
                     g["dfinal_state"])
    names = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "init_state": "dinit_state"}
    for leaf, gname in names.items():
        assert torch.equal(leaves[leaf].grad, direct[gname]), leaf


def test_full_size_layer_on_sampled_tokens(cuda_device):
    # the 2.7B-layer shape (b4, T 2048, H 80, P 64, N 128, G 1, Q 256, bf16): the whole backward on the
    # GPU, checked at sampled tokens of two batch rows against the explicit-sum oracle, dD against its
    # plain sum and dA against its definition from the checked ddt
    w = WORKLOADS["mamba2_2p7b_layer"]
    inp = workload_inputs(w)
    grads = make_output_grads(w.batch, w.T, w.H, w.P, w.N, w.dtype, seed=w.seed, with_dfinal=True)
    got = _run(inp, grads, w.Q, cuda_device)
    toks = [0, 1, 255, 256, 1029, 2047]
    for b in (0, 3):
        ref = oracle.ssd_ref_bwd_at(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], grads["dy"], b,
                                    toks, init_state=inp["init_state"], dfinal_state=grads["dfinal_state"])
        for name in ("dx", "dB", "dC", "ddt"):
            _check(name, got[name][b, toks], ref[name], w.dtype)
    dy, x = grads["dy"].double().numpy(), inp["x"].double().numpy()
    _check("dD", got["dD"], np.einsum("bthp,bthp->h", dy, x), w.dtype)
    dt, A = inp["dt"].double().numpy(), inp["A"].double().numpy()
    _check("dA", got["dA"], np.einsum("bth,bth->h", dt, got["ddt"].astype(np.float64) / A), w.dtype)


def test_backward_replays_from_a_cuda_graph(cuda_device):
    # a training step captured once and replayed: same launches, same gradients
    from structured_state_space_ssd_b200.ssd import ssd_bwd_workspace_bytes
    inp = make_inputs(2, 600, 8, 64, 128, 2, "bf16", seed=45, with_init=True)
    grads = make_output_grads(2, 600, 8, 64, 128, "bf16", seed=45, with_dfinal=True)
    d, g = _to(cuda_device, inp), _to(cuda_device, grads)
    ws = torch.empty(ssd_bwd_workspace_bytes(2, 600, 8, 64, 2, 128, 256, torch.bfloat16), dtype=torch.uint8,
                     device=cuda_device)

    def bwd():
        return ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], g["dy"], 256, d["init_state"],
                       g["dfinal_state"], workspace=ws, stream=torch.cuda.current_stream(cuda_device))

    eager = {k: v.clone() for k, v in bwd().items()}
    torch.cuda.synchronize(cuda_device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = bwd()
    for _ in range(2):
        for v in out.values():
            v.zero_()
        graph.replay()
        torch.cuda.synchronize(cuda_device)
        for k, v in eager.items():
            assert torch.equal(out[k], v), k
    del graph


@pytest.mark.parametrize("split", [300, 512])
def test_backward_of_a_split_sequence_matches_the_whole(split, cuda_device):
    # chain rule across a cut at token `split` (inside a chunk, or on a chunk boundary): the second part's
    # backward from the first part's final state hands its initial-state gradient to the first part as
    # its final-state gradient; per-token gradients concatenate, dA and dD add
    b, T, H, P, N, G, Q = 2, 900, 4, 64, 128, 2, 256
    inp = make_inputs(b, T, H, P, N, G, "f32", seed=46, with_init=True)
    grads = make_output_grads(b, T, H, P, N, "f32", seed=46, with_dfinal=True)
    d, g = _to(cuda_device, inp), _to(cuda_device, grads)
    full = ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], g["dy"], Q, d["init_state"], g["dfinal_state"])

    def part(lo, hi):
        return {k: d[k][:, lo:hi].contiguous() for k in ("x", "dt", "B", "C")}, g["dy"][:, lo:hi].contiguous()

    p1, dy1 = part(0, split)
    p2, dy2 = part(split, T)
    _, fin1 = ssd_fwd(p1["x"], p1["dt"], d["A"], p1["B"], p1["C"], d["D"], Q, d["init_state"])
    g2 = ssd_bwd(p2["x"], p2["dt"], d["A"], p2["B"], p2["C"], d["D"], dy2, Q, fin1, g["dfinal_state"])
    g1 = ssd_bwd(p1["x"], p1["dt"], d["A"], p1["B"], p1["C"], d["D"], dy1, Q, d["init_state"], g2["dinit_state"])
    torch.cuda.synchronize(cuda_device)
    for name in ("dx", "ddt", "dB", "dC"):
        joined = torch.cat([g1[name], g2[name]], dim=1)
        _check(name, joined.cpu().numpy(), full[name].double().cpu().numpy(), "f32")
    for name in ("dA", "dD"):
        _check(name, (g1[name] + g2[name]).cpu().numpy(), full[name].double().cpu().numpy(), "f32")
    _check("dinit_state", g1["dinit_state"].cpu().numpy(), full["dinit_state"].double().cpu().numpy(), "f32")


def test_status_word_is_clear_after_a_tensor_core_backward(cuda_device):
    import ctypes
    from structured_state_space_ssd_b200 import ssd as S
    inp = make_inputs(1, 600, 4, 64, 128, 2, "bf16", seed=91, with_init=True)
    grads = make_output_grads(1, 600, 4, 64, 128, "bf16", seed=91, with_dfinal=True)
    d, g = _to(cuda_device, inp), _to(cuda_device, grads)
    ws = torch.empty(S.ssd_bwd_workspace_bytes(1, 600, 4, 64, 2, 128, 256, torch.bfloat16), dtype=torch.uint8,
                     device=cuda_device)
    ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], g["dy"], 256, d["init_state"], g["dfinal_state"],
            workspace=ws)
    stream = torch.cuda.current_stream(cuda_device)
    assert S.load().ssd_bwd_check(ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(stream.cuda_stream)) == 0
    assert S.load().ssd_bwd_check(None, ctypes.c_void_p(stream.cuda_stream)) == 1
