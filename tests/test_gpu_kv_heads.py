"""Decode over a range of KV heads (lrkv_attn_decode_kv_heads), the building
block of splitting one workload's heads over GPUs.

A shard's K/V view holds only its heads; q, B and out are the whole problem's.
Where every CTA of both launches holds at most one key tile (the keys of each
(session, KV head) are then split the same way whatever the number of heads),
a shard's rows equal the same rows of the whole call bit for bit; in general
they match the fp64 oracle within the stated tolerance.  The shards of a plan
(bench.kv_head_shard_plan) together write every output row exactly once."""

import pytest
import torch

import bench
import lora_shared_kv_b200 as lrkv
from gpu_util import assert_parity, decode_oracle, to_np
from workloads.gen import _normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dense(seed, S, N, Hq, Hkv, d, r, L, mode=lrkv.BASE_SHARED):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = _normal((S, N, Hq, d), 1.0, g, DEV)
    k = _normal((S, Hkv, L, d), 1.0, g, DEV)
    v = _normal((S, Hkv, L, d), 1.0, g, DEV)
    u = _normal((S, N if mode == lrkv.BASE_SHARED else 1, L, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), 0.05, g, DEV)
    offs = torch.randint(0, L, (S, N), generator=g, device=DEV, dtype=torch.int32)
    seq = torch.full((S,), L, dtype=torch.int32, device=DEV)
    return q, k, v, u, b, offs, seq


def test_shard_equals_whole_call_bitwise_when_the_key_split_cannot_move():
    S, N, Hq, Hkv, d, r, L = 2, 2, 8, 4, 128, 16, 1000   # 8 items x 16 tiles = 128 tiles <= 148 CTAs
    q, k, v, u, b, offs, seq = _dense(41, S, N, Hq, Hkv, d, r, L)
    prob = lrkv.make_problem(S, N, Hq, Hkv, d, r, lrkv.BASE_SHARED)
    ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, L), dtype=torch.uint8, device=DEV)
    whole = torch.empty_like(q)
    lrkv.lrkv_attn_decode(prob, q, lrkv.kv_view_dense(k, v), seq, L, u, b, offs, whole, ws)
    G = Hq // Hkv
    for g0, ng in [(0, 1), (1, 2), (3, 1), (0, 4)]:
        wsh = torch.zeros(lrkv.lrkv_decode_kv_heads_workspace_bytes(prob, ng, L), dtype=torch.uint8, device=DEV)
        out = torch.full_like(q, float("nan"))
        kv = lrkv.kv_view_dense(k[:, g0:g0 + ng], v[:, g0:g0 + ng])
        lrkv.lrkv_attn_decode_kv_heads(prob, g0, ng, q, kv, seq, L, u, b, offs, out, wsh)
        torch.cuda.synchronize()
        assert lrkv.lrkv_query_device_status(wsh) == ("LRKV_OK", 0)
        heads = slice(g0 * G, (g0 + ng) * G)
        assert torch.equal(out[:, :, heads], whole[:, :, heads]), (g0, ng)
        rest = torch.ones(Hq, dtype=torch.bool)
        rest[heads] = False
        assert torch.isnan(out[:, :, rest].float()).all()  # other heads are not written


def test_plan_shards_of_a_paged_workload_match_the_oracle():
    g = torch.Generator(device=DEV)
    g.manual_seed(42)
    S, N, Hq, Hkv, d, r, L = 2, 4, 16, 8, 128, 16, 4096
    n_lp = L // 64
    q = _normal((S, N, Hq, d), 1.0, g, DEV)
    kp = _normal((S * n_lp, Hkv, 64, d), 1.0, g, DEV)
    vp = _normal((S * n_lp, Hkv, 64, d), 1.0, g, DEV)
    table = torch.randperm(S * n_lp, generator=g, device=DEV).to(torch.int32).view(S, n_lp).contiguous()
    u = _normal((S, N, L, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), 0.05, g, DEV)
    offs = torch.randint(L // 2, L, (S, N), generator=g, device=DEV, dtype=torch.int32)
    seq = torch.tensor([L, L - 100], dtype=torch.int32, device=DEV)
    out = torch.full_like(q, float("nan"))
    plan = bench.kv_head_shard_plan(S, Hkv, 3)  # three ranks: head ranges cut inside a session
    assert any(ng < Hkv for blocks in plan for (_, _, _, ng) in blocks)
    for blocks in plan:
        for (s0, ns, g0, ng) in blocks:
            prob = lrkv.make_problem(ns, N, Hq, Hkv, d, r, lrkv.BASE_SHARED)
            ws = torch.zeros(lrkv.lrkv_decode_kv_heads_workspace_bytes(prob, ng, L), dtype=torch.uint8, device=DEV)
            kv = lrkv.kv_view_paged(kp[:, g0:g0 + ng], vp[:, g0:g0 + ng], table[s0:s0 + ns])
            lrkv.lrkv_attn_decode_kv_heads(prob, g0, ng, q[s0:s0 + ns], kv, seq[s0:s0 + ns], L, u[s0:s0 + ns], b,
                                           offs[s0:s0 + ns], out[s0:s0 + ns], ws)
            torch.cuda.synchronize()
            assert lrkv.lrkv_query_device_status(ws) == ("LRKV_OK", 0)
    assert torch.isfinite(out.float()).all()  # every row written by exactly one shard
    ref = decode_oracle(q, kp, vp, u, b, offs, seq, lrkv.BASE_SHARED, page_table=table)
    assert_parity(to_np(out), ref, "kv-head shards")


def test_head_range_errors():
    q, k, v, u, b, offs, seq = _dense(43, 1, 2, 4, 2, 64, 8, 128)
    prob = lrkv.make_problem(1, 2, 4, 2, 64, 8, lrkv.BASE_SHARED)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    kv = lrkv.kv_view_dense(k, v)
    for g0, ng in [(-1, 1), (0, 0), (1, 2), (2, 1)]:
        with pytest.raises(lrkv.LrkvError) as ei:
            lrkv.lrkv_attn_decode_kv_heads(prob, g0, ng, q, kv, seq, 128, u, b, offs, torch.empty_like(q), ws)
        assert ei.value.name == "LRKV_ERR_INVALID_ARGUMENT"
