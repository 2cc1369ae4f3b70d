"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, no GPU.

The SSD forward partitions over batch and heads with no exchange, so each
rank runs its own seeded batch; the only collectives are the barriers and the
max-reduction of the timings.  These tests run that logic as world-size-2
gloo processes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from structured_state_space_ssd_b200.inputs import WORKLOADS, Workload


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("t", 2, 64, 4, 8, 8, 2, 32, "bf16", 77, True)
        inp = bench.rank_inputs(w, rank)
        local_ms = 1.0 + 2.5 * rank
        job_ms = bench.max_over_ranks(local_ms)
        dist.barrier()
        out[rank] = (float(inp["x"].float().sum()), job_ms, bench.job_tokens_per_s(w, world, job_ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_distinct_batches():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    (x0, t0, v0), (x1, t1, v1) = res[0], res[1]
    assert x0 != x1                          # each rank processes its own batch
    assert t0 == t1 == 3.5                   # every rank reports the slowest rank's time
    assert v0 == v1 == 2 * 2 * 64 / 3.5e-3   # tokens of both ranks over that time


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(4.25) == 4.25
    w = WORKLOADS["mamba2_2p7b_layer"]
    assert bench.job_tokens_per_s(w, 1, 1.0) == w.tokens / 1e-3
    assert bench.rank_inputs(WORKLOADS["tiny_f32"], 0)["x"].shape == (1, 256, 2, 16)


def _exchange_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from structured_state_space_ssd_b200.ssd import exchange_shard_states
        fin0 = torch.full((2, 3, 4, 5), float(rank + 1))   # [b, H, P, N]
        total = torch.full((2, 3), -0.5 * (rank + 1))      # [b, H]
        fin0_all, total_all = exchange_shard_states(fin0, total)
        out[rank] = (fin0_all[:, 0, 0, 0, 0].tolist(), total_all[:, 0, 0].tolist(), tuple(fin0_all.shape))
    finally:
        dist.destroy_process_group()


def test_sequence_split_exchange_stacks_states_in_rank_order():
    # the one collective of the sequence split: every rank sees every shard's state, shard k at index k
    world = 3
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_exchange_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1, 2}
    for rank in range(world):
        fins, totals, shape = res[rank]
        assert fins == [1.0, 2.0, 3.0]
        assert totals == [-0.5, -1.0, -1.5]
        assert shape == (3, 2, 3, 4, 5)
