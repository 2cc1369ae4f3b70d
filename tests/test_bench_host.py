"""Host-side checks of bench.py's bookkeeping (no GPU): the algorithmic work it divides by."""
import bench
from structured_state_space_ssd_b200.inputs import WORKLOADS


def test_forward_algorithmic_work_matches_the_block_count():
    # the pages' block-decomposition count, as tabulated for these shapes: 185.1 MB and 43.53 GFLOP for
    # the 2.7B layer, 2175.8 MB and 481.44 GFLOP for the 131k-token sequence with initial state
    b, f, _ = bench.algorithmic(WORKLOADS["mamba2_2p7b_layer"])
    assert b == 185_074_304 and f == 43_528_486_912
    b, f, _ = bench.algorithmic(WORKLOADS["long_131k"])
    assert b == 2_175_795_584 and f == 481_438_990_336


def test_forward_stage_work_adds_up():
    # the CUDA-core path's stage FLOPs (cumsum and state passing count none) sum to the pass total
    # less the 2NPH term of the state passing, which the stage list books as bytes
    w = WORKLOADS["mamba2_130m_layer"]
    _, flops, st = bench.algorithmic(w)
    staged = st["ssd_chunk_state"][1] + st["ssd_chunk_scan"][1]
    assert flops - staged == w.batch * w.nc * 2 * w.N * w.P * w.H


def test_backward_block_count():
    # per (batch, chunk) at Q 256, N 128, P 64, H 80, G 1: C B^T 16.8 M, two Q x Q x P products 2 x 671 M,
    # two Q x Q x N products 2 x 1342 M, five state products 5 x 336 M -> 183.1 GFLOP over 32 (batch, chunk)
    w = WORKLOADS["mamba2_2p7b_layer"]
    Q, N, P, H = 256, 128, 64, 80
    per = 2 * Q * Q * N + 2 * 2 * Q * Q * P * H + 2 * 2 * Q * Q * N * H + 5 * 2 * Q * N * P * H
    assert bench.backward_alg_flops(w) == 32 * per == 183_072_980_992


def test_traffic_is_reported_only_for_the_captured_kernel_source(tmp_path, monkeypatch):
    # profiles/traffic.json ties each DRAM figure to the SHA-256 of the kernel source it was captured from;
    # any other source (a changed kernel) reads None until it is captured again
    import hashlib
    import json
    src_dir = tmp_path / "structured_state_space_ssd_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    kernel = src_dir / "k.cu"
    kernel.write_text("// captured version\n")
    digest = hashlib.sha256(kernel.read_bytes()).hexdigest()
    entry = {"bytes": 123456, "source": "csrc/k.cu", "sha256": digest}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"wl": {"kern": entry}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))

    class W:
        name = "wl"

    assert bench._traffic_from_profiles("kern", W) == 123456
    assert bench._traffic_from_profiles("other", W) is None
    kernel.write_text("// changed since the capture\n")
    assert bench._traffic_from_profiles("kern", W) is None
