"""The bench's multi-rank host logic on CPU with two gloo ranks.

Each rank holds its own sessions (distinct seeds), no collective touches the
data path, and the step time reported is the slowest rank's."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from workloads import CONFIGS, make_decode_inputs
        from workloads.gen import seed_for
        cfg = CONFIGS["cfg1"]
        inp = make_decode_inputs(cfg, device="cpu", seed=seed_for(cfg) + bench.rank_seed_offset(rank))
        checksum = float(inp.layers[0].q.float().sum())
        my_ms = 1.0 + rank          # rank 1 is the slower one
        ms = bench.max_over_ranks(my_ms)
        value = bench.job_throughput(cfg.queries_per_step, world, ms)
        q.put((rank, checksum, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_sessions_and_take_the_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    (r0, c0, ms0, v0), (r1, c1, ms1, v1) = res
    assert c0 != c1                       # each rank drew its own sessions
    assert ms0 == ms1 == 2.0              # both see the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 2 / 2e-3)   # cfg1: 2 queries per rank, 2 ranks, 2 ms


def test_single_process_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(96, 1, 2.0) == pytest.approx(48000.0)
