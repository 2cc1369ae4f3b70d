"""Benchmark of the SSD layer forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one full SSD forward (every stage kernel) over one batch of the
workload's synthetic inputs, resident in HBM.  Each step is timed on the
launching stream by events the library records around its own kernels
(``ssd_fwd_timed``); L2 is flushed (a 256 MiB write) between steps, outside
the timed spans.  ``value`` is tokens/s over all ranks: sum of tokens ÷ the
max over ranks of the K-step time.  ``e2e`` repeats the measurement through
the same public call with the inputs copied in from pinned host memory and y
plus final_state copied back inside the timed region.

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch of
the workload (independent sequences, no collective on the data path), so
scaling is weak.  The only collectives are the barriers and the max-reduction
of the timings.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), on a
bounded sample of (batch, head) sequences per step, and prints the same line
with ``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSD fwd tokens/s and TFLOP/s (% of roofline) at Mamba-2-2.7B layer shape"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
N_SM = 148


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-workloads", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# Algorithmic work (block-decomposition count of the pages' cost analysis)
# ---------------------------------------------------------------------------
def algorithmic(w):
    """Per-call algorithmic bytes and FLOPs of the whole pass and of each stage.

    Bytes: x, B, C (input dtype), dt, A, D, init (fp32) read; y (input dtype)
    and final_state (fp32) written; intermediates excluded.  FLOPs per
    (batch, chunk): 2Q^2 N G (C B^T, once per group) + 2Q^2 P H (masked X
    product over the full QxQ block) + 2QNP H (chunk states) + 2QNP H
    (inter-chunk output) + 2NP H (state passing).
    """
    es = 2 if w.dtype == "bf16" else 4
    b, T, H, P, N, G, Q, nc = w.batch, w.T, w.H, w.P, w.N, w.G, w.Q, w.nc
    state = 4 * b * H * P * N
    bytes_ = (es * b * T * H * P * 2 + es * b * T * G * N * 2 + 4 * b * T * H + 8 * H
              + state * (2 if w.with_init else 1))
    per_chunk = 2 * Q * Q * N * G + 2 * Q * Q * P * H + 4 * Q * N * P * H + 2 * N * P * H
    flops = b * nc * per_chunk
    stages = {
        "ssd_fused": ("pass", (bytes_, flops)),
        "ssd_chunk_cumsum": ("hbm", 4 * b * T * H + 4 * H + 4 * b * H * nc * Q),
        "ssd_chunk_state": ("flop", b * nc * 2 * Q * N * P * H),
        "ssd_state_passing": ("hbm", 2 * 4 * b * nc * H * P * N + state * (2 if w.with_init else 1)),
        "ssd_chunk_scan": ("flop", b * nc * (2 * Q * Q * N * G + 2 * Q * Q * P * H + 2 * Q * N * P * H)),
    }
    return bytes_, flops, stages


# ---------------------------------------------------------------------------
# Clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (the baseline, and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_time(inp, w, pairs):
    import oracle
    t0 = time.perf_counter()
    oracle.ssd_ref_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                       init_state=inp["init_state"], pairs=pairs)
    return time.perf_counter() - t0


def cpu_baseline(inp, w, budget_pairs=None):
    """Time the oracle on a bounded set of (batch, head) sequences; tokens/s equivalent."""
    import oracle
    allpairs = [(b, h) for b in range(w.batch) for h in range(w.H)]
    cost = w.T * w.P * w.N  # per sequence
    if budget_pairs is None:
        # about 40 core-seconds at the oracle's ~0.5 GFLOP/s per core
        budget_pairs = max(1, int(40 * 0.5e9 / (4 * cost)))
    step = max(1, len(allpairs) // budget_pairs)
    pairs = allpairs[::step][:budget_pairs]
    # repeat the sample until about 10 s of wall time have been spent (the oracle is faster on some hosts
    # than the estimate above), at most 100 passes
    secs, passes = 0.0, 0
    while passes < 100 and (passes == 0 or secs < 10.0):
        secs += oracle_sample_time(inp, w, pairs)
        passes += 1
    tokens = passes * len(pairs) * w.T / w.H  # a sequence is one head's share of T tokens
    return {"value": tokens / secs, "unit": "tokens/s", "cores": oracle.default_threads(), "kind": "oracle",
            "sample": f"{len(pairs)} of {len(allpairs)} (batch, head) sequences of {w.name}, all {w.T} tokens, "
                      f"fp64, {passes} passes, {secs:.2f} s wall"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from structured_state_space_ssd_b200.inputs import workload_inputs
    import oracle
    inp = workload_inputs(w)
    cores = oracle.default_threads()
    allpairs = [(b, h) for b in range(w.batch) for h in range(w.H)]
    per_step = max(1, min(len(allpairs), 2 * cores))
    times = []
    for k in range(args.warmup + args.steps):
        pairs = [allpairs[(k * per_step + i) % len(allpairs)] for i in range(per_step)]
        t = oracle_sample_time(inp, w, pairs)
        if k >= args.warmup:
            times.append(t)
    tok = per_step * w.T / w.H
    value = tok * len(times) / sum(times)
    sample = (f"{per_step} (batch, head) sequences of {w.name} per step (all {w.T} tokens each), fp64, "
              f"{cores} threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Rank plumbing (one process per GPU; no collective on the data path)
# ---------------------------------------------------------------------------
def rank_inputs(w, rank: int):
    """Inputs of this rank's batch: the workload's own seed on rank 0, a distinct seed elsewhere."""
    from structured_state_space_ssd_b200.inputs import make_inputs, workload_inputs
    if rank == 0:
        return workload_inputs(w)
    return make_inputs(w.batch, w.T, w.H, w.P, w.N, w.G, w.dtype, w.seed + 7919 * rank, w.with_init)


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(w, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes one batch of the workload per step."""
    return w.tokens * world / (ms_per_step * 1e-3)


def config_of(w, n):
    return {"workload": w.name, "batch": w.batch, "seq_len": w.T, "heads": w.H, "head_dim": w.P,
            "state_dim": w.N, "groups": w.G, "chunk": w.Q, "init_state": w.with_init,
            "parallelism": f"replicas{n}" if n > 1 else "single", "l2": "flushed (256 MiB write) between steps"}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------
def main():
    args = parse()
    from structured_state_space_ssd_b200.inputs import HEADLINE, WORKLOADS
    w = WORKLOADS[args.workload or HEADLINE]
    if args.impl == "reference":
        run_reference(args, w)
        return

    import torch
    import torch.distributed as dist
    from structured_state_space_ssd_b200 import ssd as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    assert args.warmup >= 3, "at least 3 warm-up steps"

    S.load()
    host = rank_inputs(w, rank)
    d = {k: (v.to(dev) if v is not None else None) for k, v in host.items()}
    y = torch.empty_like(d["x"])
    fin = torch.empty((w.batch, w.H, w.P, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(S.ssd_fwd_workspace_bytes(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, d["x"].dtype),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = S.ssd_fwd_stage_names(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, d["x"].dtype)

    def step(stage_ms=None):
        S.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], w.Q, d["init_state"], y=y, final_state=fin,
                  workspace=ws, stream=stream, stage_ms=stage_ms)

    gpu_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local] \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else str(local)
    sampler = ClockSampler(gpu_index)
    sampler.start()
    time.sleep(0.2)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    per_step = []
    per_stage = [[] for _ in names]
    for _ in range(args.steps):
        flush.zero_()
        ms = []
        step(ms)
        for i in range(len(names)):
            per_stage[i].append(ms[i])
        per_step.append(ms[-1])
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(sum(per_step), dev)
    ms_per_step = total_ms / args.steps
    tokens = w.tokens * world
    value = job_tokens_per_s(w, world, ms_per_step)

    # --- end to end: pinned host inputs in, y and final_state out, every step.  As a serving or training
    # loop would run it: two device buffer sets, the inputs copied in on one stream and the outputs out on
    # another, so that step k's copies overlap the compute of its neighbours (the link carries both
    # directions at once); every step's copies are inside the timed region.
    e2e_steps = args.e2e_steps or args.steps
    pinned = {k: (v.pin_memory() if v is not None else None) for k, v in host.items()}
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    fin_host = torch.empty(fin.shape, dtype=fin.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values() if v is not None)
    d2h = y_host.numel() * y_host.element_size() + fin_host.numel() * fin_host.element_size()
    d2 = {k: (torch.empty_like(v) if v is not None else None) for k, v in d.items()}
    sets = [(d, y, fin), (d2, torch.empty_like(y), torch.empty_like(fin))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(nsteps):
        ev = [[torch.cuda.Event() for _ in range(3)] for _ in range(nsteps)]  # copied in, computed, copied out
        for k in range(nsteps):
            dk, yk, fk = sets[k % 2]
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(ev[k - 2][1])  # step k-2 has read this set's inputs
                for name, v in pinned.items():
                    if v is not None:
                        dk[name].copy_(v, non_blocking=True)
                ev[k][0].record(s_in)
            stream.wait_event(ev[k][0])
            if k >= 2:
                stream.wait_event(ev[k - 2][2])  # step k-2's outputs have left this set
            S.ssd_fwd(dk["x"], dk["dt"], dk["A"], dk["B"], dk["C"], dk["D"], w.Q, dk["init_state"], y=yk,
                      final_state=fk, workspace=ws, stream=stream)
            ev[k][1].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev[k][1])
                y_host.copy_(yk, non_blocking=True)
                fin_host.copy_(fk, non_blocking=True)
                ev[k][2].record(s_out)

    e2e_run(args.warmup)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    e2e_run(e2e_steps)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    if world > 1:
        dist.barrier()

    if rank == 0:
        peaks, peak_src = load_peaks()
        alg_bytes, alg_flops, stages = algorithmic(w)
        stage_avg = {n: sum(v) / len(v) for n, v in zip(names, per_stage)}
        dom = max(stage_avg, key=stage_avg.get)
        kind, amount = stages[dom]
        dom_ms = stage_avg[dom]
        both = None
        if kind == "pass":
            # bytes and FLOPs both matter: the bound is the slower of the two at peak
            fb, ff = amount
            t_mem, t_tc = fb / (peaks["hbm_gbs"] * 1e9), ff / (peaks["bf16_tflops"] * 1e12)
            both = {"hbm_GBps": fb / (dom_ms * 1e-3) / 1e9, "hbm_frac": fb / (dom_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "tensor_TFLOPs": ff / (dom_ms * 1e-3) / 1e12,
                    "tensor_frac": ff / (dom_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                    "alg_bytes": fb, "alg_flops": ff}
            kind, amount = ("hbm", fb) if t_mem >= t_tc else ("tensor", ff)
        if kind == "hbm":
            roof = {"bound": "hbm", "achieved": amount / (dom_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s"}
        else:
            if both is not None:
                roof = {"bound": "tensor", "achieved": amount / (dom_ms * 1e-3) / 1e12,
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
            else:
                fp32_peak = N_SM * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
                roof = {"bound": "alu", "achieved": amount / (dom_ms * 1e-3) / 1e12, "peak": fp32_peak,
                        "unit": "TFLOP/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = _traffic_from_profiles(dom, w)
        roof["kernel"] = dom
        if both is not None:
            roof["both"] = both
        roof["peak_source"] = f"{peak_src} (burst)" if roof["bound"] != "alu" else \
            "derived: 148 SMs x 128 fp32 FMA/clk x 2 x max SM clock"
        t_roof = max(alg_bytes / (peaks["hbm_gbs"] * 1e9), alg_flops / (peaks["bf16_tflops"] * 1e12))
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1)/softplus inputs, see inputs.py)",
            "config": config_of(w, world),
            "tflops": alg_flops * world / (ms_per_step * 1e-3) / 1e12,
            "pass_roofline": {"alg_bytes": alg_bytes, "alg_flops": alg_flops, "roofline_ms": t_roof * 1e3,
                              "frac": t_roof * 1e3 / ms_per_step, "peaks": peak_src},
            "roofline": roof,
            "kernels_ms": stage_avg,
            "clocks": clocks,
            "e2e": {"value": tokens * e2e_steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / e2e_steps,
                    "pipelined": "two device buffer sets; inputs in, compute and outputs out of neighbouring "
                                 "steps overlap on three streams"},
            # the main launches, plus the fused path's workspace-clear kernel (timed within its first stage)
            "gpu_launches": (S.ssd_fwd_launch_count(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, d["x"].dtype)
                             + (1 if names[0].startswith("ssd_fused") else 0)) * args.steps,
        }
        if world == 1 and not args.no_workloads:
            line["workloads"] = measure_workloads(w, dev, stream, flush, peaks)
        line["decode_step"] = measure_decode(w, host, dev, stream, flush, peaks)
        line["gate_norm"] = measure_gate_norm(w, y, dev, stream, flush, peaks)
        line["gated_forward"] = measure_gated(w, d, dev, stream, flush, line["gate_norm"]["us_per_launch"],
                                              ms_per_step)
        line["backward"] = measure_backward(w, d, dev, stream, flush, peaks)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(host, w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_workloads(headline, dev, stream, flush, peaks, steps=10, warmup=3):
    """Every other bf16 workload of the configuration list, timed like the headline (L2 flushed between
    steps, CUDA events recorded by the library around its kernels).  Their inputs are drawn on the GPU
    (same distributions as the seeded CPU draws the parity tests use): only time is measured here."""
    import torch
    from structured_state_space_ssd_b200 import ssd as S
    from structured_state_space_ssd_b200.inputs import WORKLOADS, make_inputs
    out = {}
    for name, w in WORKLOADS.items():
        if name == headline.name or w.dtype != "bf16":
            continue
        d = make_inputs(w.batch, w.T, w.H, w.P, w.N, w.G, w.dtype, w.seed, w.with_init, device=str(dev))
        y = torch.empty_like(d["x"])
        fin = torch.empty((w.batch, w.H, w.P, w.N), dtype=torch.float32, device=dev)
        ws = torch.empty(S.ssd_fwd_workspace_bytes(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, d["x"].dtype),
                         dtype=torch.uint8, device=dev)
        names = S.ssd_fwd_stage_names(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, d["x"].dtype)
        per_step, per_stage = [], [[] for _ in names]
        for k in range(warmup + steps):
            flush.zero_()
            ms = []
            S.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], w.Q, d["init_state"], y=y, final_state=fin,
                      workspace=ws, stream=stream, stage_ms=ms)
            if k >= warmup:
                per_step.append(ms[-1])
                for i in range(len(names)):
                    per_stage[i].append(ms[i])
        ms_step = sum(per_step) / len(per_step)
        alg_bytes, alg_flops, _ = algorithmic(w)
        t_roof = max(alg_bytes / (peaks["hbm_gbs"] * 1e9), alg_flops / (peaks["bf16_tflops"] * 1e12))
        out[name] = {"ms_per_step": ms_step, "tokens_per_s": w.tokens / (ms_step * 1e-3),
                     "tflops": alg_flops / (ms_step * 1e-3) / 1e12,
                     "pass_roofline": {"roofline_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_step},
                     "kernels_ms": {n: sum(v) / len(v) for n, v in zip(names, per_stage)}}
        del d, y, fin, ws
        torch.cuda.empty_cache()
    return out


def measure_decode(w, host, dev, stream, flush, peaks, steps=50, resident_steps=200):
    """The decode step (one token of the recurrence, ssd_step) on the workload's batch, heads and state.

    Each step reads and writes the whole fp32 state, so it is HBM-bound when the state is cold
    (L2 flushed before every timed step) and L2-bound inside a decode loop that keeps it resident.
    """
    import torch
    from structured_state_space_ssd_b200 import ssd as S
    b, H, P, G, N = w.batch, w.H, w.P, w.G, w.N
    gen = torch.Generator().manual_seed(w.seed + 99)
    state = torch.randn((b, H, P, N), generator=gen).to(dev)
    x, dt, B, C = (host[k][:, 0].contiguous().to(dev) for k in ("x", "dt", "B", "C"))
    A, D = host["A"].to(dev), host["D"].to(dev)
    y = torch.empty_like(x)
    es = x.element_size()
    alg = 2 * state.numel() * 4 + 2 * x.numel() * es + 2 * B.numel() * es + dt.numel() * 4 + 2 * H * 4

    def one():
        S.ssd_step(state, x, dt, A, B, C, D, y=y, stream=stream)

    for _ in range(5):
        flush.zero_()
        one()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        one()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    cold_ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    # a decode loop as a user runs it: the steps captured once in a CUDA graph and replayed, so that
    # the host does not pace the launches
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cap = torch.cuda.current_stream(dev)
        for _ in range(resident_steps):
            S.ssd_step(state, x, dt, A, B, C, D, y=y, stream=cap)
    graph.replay()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    graph.replay()
    r1.record(stream)
    torch.cuda.synchronize(dev)
    warm_ms = r0.elapsed_time(r1) / resident_steps
    del graph
    gbps = alg / (cold_ms * 1e-3) / 1e9
    return {"state_shape": [b, H, P, N], "dtype": w.dtype, "alg_bytes": alg,
            "us_per_step_cold": cold_ms * 1e3, "GBps_cold": gbps, "frac_of_hbm": gbps / peaks["hbm_gbs"],
            "us_per_step_l2_resident": warm_ms * 1e3, "l2_resident_loop": f"{resident_steps} steps in one CUDA graph",
            "GBps_l2_resident": alg / (warm_ms * 1e-3) / 1e9, "launches_per_step": 1}


def measure_gate_norm(w, y, dev, stream, flush, peaks, steps=20):
    """The block's step after the layer (Swish gate by z, GroupNorm with a group per head) on this
    workload's output y, L2 flushed before each launch: one read of y and z, one write."""
    import torch
    from structured_state_space_ssd_b200 import ssd as S
    gen = torch.Generator().manual_seed(w.seed + 7)
    yv = y.view(-1, w.H * w.P)  # per token: all heads' channels
    z = torch.randn(tuple(yv.shape), generator=gen).to(y.dtype).to(dev)
    out = torch.empty_like(yv)
    alg = 3 * y.numel() * y.element_size()

    def one():
        S.ssd_gate_norm(yv, z, w.H, 1e-5, out=out, stream=stream)

    for _ in range(3):
        flush.zero_()
        one()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        one()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    gbps = alg / (ms * 1e-3) / 1e9
    return {"rows": y.numel() // (w.H * w.P), "channels": w.H * w.P, "ngroups": w.H, "dtype": w.dtype,
            "alg_bytes": alg, "us_per_launch": ms * 1e3, "GBps": gbps, "frac_of_hbm": gbps / peaks["hbm_gbs"]}


def measure_gated(w, d, dev, stream, flush, gate_us, fwd_ms, steps=20):
    """The forward with the gate and the per-head GroupNorm in the fused kernel's drain (ssd_fwd_gated) on
    this workload, L2 flushed before each call, against the forward followed by the gate kernel (the
    step line's ms_per_step plus the gate_norm object's time)."""
    import torch
    from structured_state_space_ssd_b200 import ssd as S
    gen = torch.Generator().manual_seed(w.seed + 11)
    z = torch.randn(tuple(d["x"].shape), generator=gen).to(d["x"].dtype).to(dev)
    wt = (torch.rand(w.H * w.P, generator=gen) + 0.5).to(dev)
    bs = torch.randn(w.H * w.P, generator=gen).to(dev)
    out = torch.empty_like(d["x"])
    fin = torch.empty((w.batch, w.H, w.P, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(S.ssd_fwd_workspace_bytes(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, d["x"].dtype),
                     dtype=torch.uint8, device=dev)

    def one():
        S.ssd_fwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], w.Q, z, d["init_state"], wt, bs, 1e-5,
                        out=out, final_state=fin, workspace=ws, stream=stream)

    for _ in range(3):
        flush.zero_()
        one()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        one()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    launches = S.load().ssd_fwd_gated_launch_count(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q,
                                                   S._dtype_code(d["x"].dtype))
    # plus the fused path's workspace-clear kernel
    if S.ssd_fwd_stage_names(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, d["x"].dtype)[0].startswith("ssd_fused"):
        launches += 1
    return {"ms_per_call": ms, "tokens_per_s": w.batch * w.T / (ms * 1e-3), "launches_per_call": launches,
            "separate_ms": fwd_ms + gate_us * 1e-3, "with": "z, norm weight and bias; one group per head"}


def backward_alg_flops(w):
    """Block-form work of the backward per call: per (batch, chunk), C B^T once per group; the masked
    Q x Q products for dx and for W = dy x^T, and those of W with C and B for dB and dC; five Q x N x P
    state products (forward and backward chunk states, the state terms of dx, dB and dC)."""
    Q, H, P, N, G = w.Q, w.H, w.P, w.N, w.G
    per_chunk = 2 * Q * Q * N * G + 2 * (2 * Q * Q * P * H) + 2 * (2 * Q * Q * N * H) + 5 * (2 * Q * N * P * H)
    return per_chunk * w.batch * w.nc


def measure_backward(w, d, dev, stream, flush, peaks, steps=5):
    """The layer's backward (ssd_bwd: every input gradient for given dy and dfinal) on this workload,
    L2 flushed before each call.  Its products (the three masked chunk scans and the chunk states) run on
    the bf16 tensor cores, so the block count is set against the measured bf16 peak; the products of the
    per-head dB, dC terms and of the chunk states are issued twice (high and low bf16 parts), which the
    block count does not include."""
    import torch
    from structured_state_space_ssd_b200 import ssd as S
    from structured_state_space_ssd_b200.inputs import make_output_grads
    g = make_output_grads(w.batch, w.T, w.H, w.P, w.N, w.dtype, seed=w.seed, with_dfinal=True)
    dy, dfin = g["dy"].to(dev), g["dfinal_state"].to(dev)
    ws = torch.empty(S.ssd_bwd_workspace_bytes(w.batch, w.T, w.H, w.P, w.G, w.N, w.Q, dy.dtype), dtype=torch.uint8,
                     device=dev)
    Q = w.Q
    alg_flops = backward_alg_flops(w)

    def one():
        S.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], dy, Q, d["init_state"], dfin, workspace=ws,
                  stream=stream)

    for _ in range(3):
        flush.zero_()
        one()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        one()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    tflops = alg_flops / (ms * 1e-3) / 1e12
    return {"ms": ms, "tokens_per_s": w.tokens / (ms * 1e-3), "alg_flops": alg_flops,
            "tflops": tflops, "bound": "tensor", "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
            "launches_per_call": 11,
            "with": "dfinal_state and init_state" if w.with_init else "dfinal_state (the workload has no init_state)"}


def _traffic_from_profiles(kernel, w):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, if one matches this workload and was
    taken on the kernel's current source (the entry records the SHA-256 of the source file it was captured
    from; a changed kernel reports None until it is captured again)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(w.name, {}).get(kernel)
    if not isinstance(e, dict):
        return None
    src = os.path.join(ROOT, "structured_state_space_ssd_b200", e.get("source", ""))
    if not os.path.isfile(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != e.get("sha256"):
            return None
    return e.get("bytes")


if __name__ == "__main__":
    main()
