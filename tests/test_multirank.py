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


@pytest.mark.parametrize("S,Hkv,world", [(4, 8, 1), (4, 8, 2), (4, 8, 4), (4, 8, 8), (4, 8, 3), (4, 8, 5),
                                         (32, 2, 8), (1, 8, 8), (3, 2, 4), (2, 8, 16)])
def test_kv_head_shard_plan_covers_every_pair_once(S, Hkv, world):
    import bench
    plan = bench.kv_head_shard_plan(S, Hkv, world)
    assert len(plan) == world
    seen = {}
    for rank, blocks in enumerate(plan):
        for (s0, ns, g0, ng) in blocks:
            assert ns >= 1 and ng >= 1 and 0 <= g0 and g0 + ng <= Hkv and 0 <= s0 and s0 + ns <= S
            assert ns == 1 or (g0 == 0 and ng == Hkv)     # several sessions only as whole sessions
            for s in range(s0, s0 + ns):
                for g in range(g0, g0 + ng):
                    assert (s, g) not in seen, (s, g)
                    seen[(s, g)] = rank
    assert sorted(seen) == [(s, g) for s in range(S) for g in range(Hkv)]
    loads = [sum(ns * ng for (_, ns, _, ng) in blocks) for blocks in plan]
    assert max(loads) - min(loads) <= 1                   # balanced to one pair


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from workloads import CONFIGS
        cfg = CONFIGS["cfg5"]
        blocks = bench.kv_head_shard_plan(cfg.S, cfg.Hkv, world)[rank]
        offs = torch.full((cfg.S, cfg.N), 40000, dtype=torch.int32)
        mine = bench.shard_layer_bytes(cfg, offs, blocks)
        total = torch.tensor([float(mine)], dtype=torch.float64)
        dist.all_reduce(total)                              # test-side sum, not a data-path collective
        ms = bench.max_over_ranks(1.0 + 0.5 * rank)
        q.put((rank, len(blocks), mine, float(total.item()), ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_the_kv_heads_of_one_workload():
    import bench
    from workloads import CONFIGS
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    cfg = CONFIGS["cfg5"]
    offs = torch.full((cfg.S, cfg.N), 40000, dtype=torch.int32)
    whole = bench.decode_layer_bytes(cfg, offs)
    # two ranks, two whole sessions each: together they move the whole workload's bytes, except that each
    # rank reads every B column of its heads (here all of them) once
    b_bytes = cfg.N * cfg.r * cfg.Hkv * cfg.d * 2
    assert [r[1] for r in res] == [1, 1]
    assert res[0][3] == res[1][3] == float(whole + b_bytes)
    assert res[0][2] == res[1][2] == (whole - b_bytes) // 2 + b_bytes
    assert res[0][4] == res[1][4] == 1.5                  # the slowest rank's time
