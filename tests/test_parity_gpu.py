"""GPU parity: libssd.so (through its C ABI) against the fp64 CPU oracle.

Small shapes are compared element by element on every output; the full
workloads are compared on sampled (batch, head) sequences, which the oracle
computes one by one (every token and channel of those sequences, plus their
final states).
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, metrics
from structured_state_space_ssd_b200 import WORKLOADS, make_inputs, workload_inputs
from structured_state_space_ssd_b200.ssd import ssd_fwd, ssd_fwd_check

pytestmark = pytest.mark.gpu


def _gpu(inp, Q, dev):
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    y, fin = ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], Q, d["init_state"])
    torch.cuda.synchronize(dev)
    return y.float().cpu().numpy(), fin.cpu().numpy()


def _oracle(inp, pairs=None):
    return oracle.ssd_ref_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                              init_state=inp["init_state"], pairs=pairs)


SMALL = [
    # batch, T, H, P, N, G, Q, dtype, init
    (1, 256, 2, 16, 16, 1, 64, "f32", False),     # the tiny fp32 workload's shape
    (2, 100, 4, 16, 16, 2, 64, "f32", True),      # ragged last chunk, grouped heads, initial state
    (1, 37, 2, 8, 8, 1, 1, "f32", True),          # Q = 1: the pure recurrence
    (1, 96, 3, 5, 7, 1, 96, "f32", False),        # one chunk, odd P and N
    (1, 1, 2, 4, 4, 2, 16, "f32", True),          # a single token
    (1, 1000, 2, 16, 16, 1, 16, "f32", True),     # 63 chunks for the state recurrence
    (1, 300, 2, 128, 256, 1, 256, "f32", True),   # largest P, N and Q, ragged
    (2, 200, 4, 1, 1, 4, 32, "f32", False),       # P = N = 1, G = H
    (2, 333, 4, 64, 128, 2, 128, "bf16", True),   # bf16, ragged, grouped
    (1, 512, 8, 64, 64, 1, 256, "bf16", False),
    (1, 700, 6, 64, 16, 3, 256, "bf16", True),    # small N, ragged
    (1, 256, 2, 64, 256, 1, 64, "bf16", False),   # largest N in bf16
    (1, 700, 4, 64, 256, 2, 256, "bf16", True),   # N = 256 on the tensor cores: two half-state launches
    (2, 333, 2, 64, 256, 1, 128, "bf16", True),   # the same with one row block per chunk, ragged
    (1, 100, 2, 64, 256, 1, 256, "bf16", True),   # ... and a single short chunk
    (1, 700, 4, 32, 128, 2, 256, "bf16", True),   # P = 32 on the tensor cores: zero-padded to 64 columns
    (2, 333, 3, 8, 64, 1, 128, "bf16", True),     # the narrowest head, one row block per chunk
    (1, 600, 2, 48, 16, 1, 256, "bf16", False),   # P = 48, small N
    (1, 700, 4, 128, 128, 2, 256, "bf16", True),  # P = 128: two launches over head-column halves
    (2, 300, 2, 128, 64, 1, 128, "bf16", True),   # the same with one row block per chunk
    (1, 520, 2, 128, 256, 1, 256, "bf16", True),  # P = 128, N = 256: four launches
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "b{}_T{}_H{}_P{}_N{}_G{}_Q{}_{}_{}".format(*c))
def test_small_shapes_match_oracle(case, cuda_device):
    batch, T, H, P, N, G, Q, dtype, init = case
    inp = make_inputs(batch, T, H, P, N, G, dtype, seed=100 + SMALL.index(case), with_init=init)
    y, fin = _gpu(inp, Q, cuda_device)
    y_ref, fin_ref = _oracle(inp)
    assert_close(y, y_ref, dtype, "y")
    assert_close(fin, fin_ref, dtype, "final_state")


@pytest.mark.parametrize("mode", ["A_zero", "zero_decay", "steep_decay"])
def test_special_decays_match_oracle(mode, cuda_device):
    inp = make_inputs(2, 300, 4, 32, 32, 2, "f32", seed=5, with_init=True)
    if mode == "A_zero":           # no decay: causal linear attention
        inp["A"] = torch.zeros_like(inp["A"])
    elif mode == "zero_decay":     # exp underflows to 0: only the diagonal term is left
        inp["A"] = torch.full_like(inp["A"], -1e8)
    else:                          # log-decays far below the fp32 exp range inside one chunk
        inp["dt"] = inp["dt"] * 300
    y, fin = _gpu(inp, 64, cuda_device)
    y_ref, fin_ref = _oracle(inp)
    assert_close(y, y_ref, "f32", "y")
    assert_close(fin, fin_ref, "f32", "final_state")


def test_empty_sequence_copies_initial_state(cuda_device):
    inp = make_inputs(2, 0, 2, 8, 8, 1, "f32", seed=1, with_init=True)
    y, fin = _gpu(inp, 64, cuda_device)
    assert y.shape == (2, 0, 2, 8)
    np.testing.assert_array_equal(fin, inp["init_state"].numpy())
    inp["init_state"] = None
    _, fin = _gpu(inp, 64, cuda_device)
    assert (fin == 0).all()


@pytest.mark.parametrize("dtype,split", [("f32", 128), ("f32", 77), ("bf16", 256), ("bf16", 301)])
def test_sequence_continuation_on_gpu(dtype, split, cuda_device):
    """[0, s) then [s, T) seeded with the first final state equals one run."""
    inp = make_inputs(1, 600, 4, 64, 64, 1, dtype, seed=9, with_init=True)
    y, fin = _gpu(inp, 128, cuda_device)
    first = {k: (v[:, :split].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    second = {k: (v[:, split:].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    ya, fa = _gpu(first, 128, cuda_device)
    second["init_state"] = torch.from_numpy(fa)
    yb, fb = _gpu(second, 128, cuda_device)
    assert_close(np.concatenate([ya, yb], axis=1), y, dtype, "y")
    assert_close(fb, fin, dtype, "final_state")


@pytest.mark.parametrize("Q", [16, 64, 128, 256])
def test_chunk_size_does_not_change_the_function(Q, cuda_device):
    inp = make_inputs(1, 512, 4, 64, 128, 1, "bf16", seed=13, with_init=True)
    y, fin = _gpu(inp, Q, cuda_device)
    y_ref, fin_ref = _oracle(inp)
    assert_close(y, y_ref, "bf16", f"y Q={Q}")
    assert_close(fin, fin_ref, "bf16", f"final_state Q={Q}")


@pytest.mark.parametrize("nc", [1, 2, 3, 5, 15, 16, 17, 31, 32, 33, 64, 129, 512])
def test_chunk_count_sweep_with_initial_state(nc, cuda_device):
    # 1 to 512 chunks of 128 tokens, the last one ragged: the inter-chunk chain with one hand-off per
    # chunk (below 32 chunks) and with look-back over 4 chunks (32 and more)
    T = nc * 128 - (37 if nc > 1 else 0)
    inp = make_inputs(1, T, 3, 64, 64, 1, "bf16", seed=500 + nc, with_init=True)
    y, fin = _gpu(inp, 128, cuda_device)
    y_ref, fin_ref = _oracle(inp)
    assert_close(y, y_ref, "bf16", f"y nc={nc}")
    assert_close(fin, fin_ref, "bf16", f"final_state nc={nc}")


@pytest.mark.parametrize("nc", [1, 2, 3, 4, 5, 7, 17, 31])
def test_chunk_count_sweep_two_row_blocks(nc, cuda_device):
    # Q = 256 below the look-back threshold: the chunk's second block owns the state and the first takes
    # S~_{c-1} as the owner's bf16 tile (three slots, reused from the fourth chunk on); the last chunk
    # ragged to two row blocks (odd nc) or one (even nc, where its only block owns it)
    T = nc * 256 - (37 if nc % 2 else 170)
    inp = make_inputs(2, T, 4, 64, 128, 2, "bf16", seed=700 + nc, with_init=True)
    y, fin = _gpu(inp, 256, cuda_device)
    y_ref, fin_ref = _oracle(inp)
    assert_close(y, y_ref, "bf16", f"y nc={nc}")
    assert_close(fin, fin_ref, "bf16", f"final_state nc={nc}")


def test_tile_hand_off_is_bitwise_identical_and_matches_oracle(cuda_device):
    # 31 chunks of 256 tokens (just under the look-back threshold) and 96 sequences in groups of 6 heads:
    # every tile slot is reused ten times with units of both sizes in flight on every SM; a tile read
    # before its store landed, or a slot overwritten before its read, shows up as a run-to-run difference
    inp = make_inputs(2, 31 * 256 - 5, 48, 64, 128, 8, "bf16", seed=23, with_init=True)
    runs = [_gpu(inp, 256, cuda_device) for _ in range(3)]
    for y, f in runs[1:]:
        assert np.array_equal(runs[0][0], y) and np.array_equal(runs[0][1], f)
    y_ref, fin_ref = _oracle(inp)
    assert_close(runs[0][0], y_ref, "bf16", "y")
    assert_close(runs[0][1], fin_ref, "bf16", "final_state")


@pytest.mark.parametrize("case", [(1, 9000, 4, 64, 128, 2, 256), (1, 8300, 2, 128, 256, 1, 256),
                                  (2, 4500, 3, 32, 64, 3, 128)],
                         ids=lambda c: "b{}_T{}_H{}_P{}_N{}_G{}_Q{}".format(*c))
def test_look_back_shapes_match_oracle(case, cuda_device):
    # long sequences with few heads: the chain uses look-back (with both column splits in the second)
    batch, T, H, P, N, G, Q = case
    inp = make_inputs(batch, T, H, P, N, G, "bf16", seed=77 + T, with_init=True)
    y, fin = _gpu(inp, Q, cuda_device)
    y_ref, fin_ref = _oracle(inp)
    assert_close(y, y_ref, "bf16", "y")
    assert_close(fin, fin_ref, "bf16", "final_state")


def test_repeated_runs_are_bitwise_identical(cuda_device):
    w = WORKLOADS["mamba2_2p7b_layer"]
    inp = workload_inputs(w)
    y1, f1 = _gpu(inp, w.Q, cuda_device)
    y2, f2 = _gpu(inp, w.Q, cuda_device)
    assert np.array_equal(y1, y2) and np.array_equal(f1, f2)


def test_repeated_runs_are_bitwise_identical_with_many_small_units(cuda_device):
    # many chunks and groups of 6 heads: units of every kind in flight on every SM at once,
    # the case where a hand-off that is not ordered shows up as run-to-run differences
    inp = make_inputs(1, 32768, 48, 64, 128, 8, "bf16", seed=21, with_init=True)
    runs = [_gpu(inp, 256, cuda_device) for _ in range(3)]
    for y, f in runs[1:]:
        assert np.array_equal(runs[0][0], y) and np.array_equal(runs[0][1], f)


def _sample_pairs(w, k):
    rng = np.random.default_rng(w.seed)
    pairs = {(0, 0), (w.batch - 1, w.H - 1)}
    while len(pairs) < min(k, w.batch * w.H):
        pairs.add((int(rng.integers(w.batch)), int(rng.integers(w.H))))
    return sorted(pairs)


def _fold_pairs(inp, w, pairs):
    """The sampled (batch, head) sequences as one oracle problem: batch 1, one head and one group each.

    Head i of the folded problem is sequence (b_i, h_i) with its own A, D, dt,
    initial state and its group's B/C, so the oracle's result for it is exactly
    that sequence's result in the full problem.
    """
    hpg = w.H // w.G
    bs = [p[0] for p in pairs]
    hs = [p[1] for p in pairs]
    gs = [h // hpg for h in hs]
    fold = {
        "x": torch.stack([inp["x"][b, :, h] for b, h in pairs], dim=1)[None],
        "dt": torch.stack([inp["dt"][b, :, h] for b, h in pairs], dim=1)[None],
        "A": inp["A"][hs], "D": inp["D"][hs],
        "B": torch.stack([inp["B"][b, :, g] for b, g in zip(bs, gs)], dim=1)[None],
        "C": torch.stack([inp["C"][b, :, g] for b, g in zip(bs, gs)], dim=1)[None],
        "init_state": None if inp["init_state"] is None else
        torch.stack([inp["init_state"][b, h] for b, h in pairs])[None],
    }
    return fold


@pytest.mark.parametrize("name", [n for n in WORKLOADS])
def test_workload_matches_oracle_on_sampled_heads(name, cuda_device):
    w = WORKLOADS[name]
    inp = workload_inputs(w)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    y, fin = ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], w.Q, d["init_state"])
    torch.cuda.synchronize(cuda_device)
    # every output is finite, not only the sampled ones
    assert bool(torch.isfinite(y).all()) and bool(torch.isfinite(fin).all())
    pairs = _sample_pairs(w, 6 if w.T > 8192 else 8)
    got_y = torch.stack([y[b, :, h] for b, h in pairs], dim=1).float().cpu().numpy()
    got_f = torch.stack([fin[b, h] for b, h in pairs]).cpu().numpy()
    del y, fin, d
    y_ref, fin_ref = _oracle(_fold_pairs(inp, w, pairs))
    assert_close(got_y, y_ref[0], w.dtype, f"{name} y")
    assert_close(got_f, fin_ref[0], w.dtype, f"{name} final_state")


def test_status_word_is_clear_after_a_run(cuda_device):
    inp = make_inputs(1, 256, 2, 16, 16, 1, "f32", seed=3)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    from structured_state_space_ssd_b200.ssd import ssd_fwd_workspace_bytes
    ws = torch.zeros(ssd_fwd_workspace_bytes(1, 256, 2, 16, 1, 16, 64, torch.float32), dtype=torch.uint8,
                     device=cuda_device)
    ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 64, None, workspace=ws)
    assert ssd_fwd_check(ws) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_replays_from_a_cuda_graph(dtype, cuda_device):
    # a serving loop captures the forward once and replays it: same launches, same results
    inp = make_inputs(2, 600, 8, 64, 128, 2, dtype, seed=31, with_init=True)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    from structured_state_space_ssd_b200.ssd import ssd_fwd_workspace_bytes
    ws = torch.empty(ssd_fwd_workspace_bytes(2, 600, 8, 64, 2, 128, 256, d["x"].dtype), dtype=torch.uint8,
                     device=cuda_device)
    y = torch.empty_like(d["x"])
    fin = torch.empty((2, 8, 64, 128), dtype=torch.float32, device=cuda_device)

    def fwd():
        ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256, d["init_state"], y=y, final_state=fin,
                workspace=ws, stream=torch.cuda.current_stream(cuda_device))

    fwd()
    torch.cuda.synchronize(cuda_device)
    y_eager, f_eager = y.clone(), fin.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fwd()
    for _ in range(2):
        y.zero_()
        fin.zero_()
        graph.replay()
        torch.cuda.synchronize(cuda_device)
        assert torch.equal(y, y_eager) and torch.equal(fin, f_eager)
    del graph
