"""Decode through the entry point that allocates nothing.

Some callers may not allocate device memory when they call attention: a
plug-in inside a serving engine whose device memory belongs to the engine's
own allocator, or a long-running server where cudaMalloc would synchronise the
device and can fail on a fragmented heap.  lrkv_attn_decode_static_scratch
serves them from one fixed scratch array inside the library.  These tests call
it through the C ABI, twice in a row (the scratch keeps the previous call's
contents), and compare each output with the fp64 oracle and with the regular
entry point that takes a caller-owned workspace, under the same tolerance as
the other decode tests.  The scratch's device-side flags are read back with
lrkv_query_static_scratch_status.
"""

import pytest
import torch

import lora_shared_kv_b200 as lrkv
from gpu_util import MAX_ABS, REL_L2, assert_parity, decode_oracle, errors, to_np
from workloads.gen import _normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(seed, S=4, N=3, Hq=12, Hkv=2, d=128, r=16, L=2048, mode=lrkv.BASE_SHARED, paged=False):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = _normal((S, N, Hq, d), 1.0, g, DEV)
    u = _normal((S, N if mode == lrkv.BASE_SHARED else 1, L, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), 0.05, g, DEV)
    offs = torch.tensor([[100, 1500, 2047, 5][:N]] * S, dtype=torch.int32, device=DEV)
    seq = torch.tensor([L, L - 1, L // 2, 77][:S], dtype=torch.int32, device=DEV)
    if not paged:
        k = _normal((S, Hkv, L, d), 1.0, g, DEV)
        v = _normal((S, Hkv, L, d), 1.0, g, DEV)
        return q, k, v, u, b, offs, seq, None
    n_lp = L // 64
    k = _normal((S * n_lp + 3, Hkv, 64, d), 1.0, g, DEV)
    v = _normal((S * n_lp + 3, Hkv, 64, d), 1.0, g, DEV)
    perm = torch.randperm(S * n_lp + 3, generator=g, device=DEV)[:S * n_lp]
    table = perm.to(torch.int32).view(S, n_lp).contiguous()
    return q, k, v, u, b, offs, seq, table


CASES = [
    dict(),                                                          # dense BaseShared, Qwen2.5-Coder heads
    dict(S=2, N=4, Hq=16, Hkv=8, L=4096, mode=lrkv.BASE_LR_SHARED, paged=True),  # paged, one shared U
]


@pytest.mark.parametrize("case", CASES, ids=["dense-shared", "paged-lrshared"])
def test_static_scratch_decode_matches_oracle_and_workspace_decode_twice(case):
    for seed in (101, 202):  # two calls in a row on different inputs
        q, k, v, u, b, offs, seq, table = _case(seed, **case)
        S, N, Hq, d = q.shape
        L = u.shape[2]
        mode = case.get("mode", lrkv.BASE_SHARED)
        prob = lrkv.make_problem(S, N, Hq, k.shape[1], d, u.shape[-1], mode)
        kv = lrkv.kv_view_dense(k, v) if table is None else lrkv.kv_view_paged(k, v, table)
        ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, L), dtype=torch.uint8, device=DEV)
        ref = torch.empty_like(q)
        lrkv.lrkv_attn_decode(prob, q, kv, seq, L, u, b, offs, ref, ws)
        got = torch.full_like(q, float("nan"))
        lrkv.lrkv_attn_decode_static_scratch(prob, q, kv, seq, L, u, b, offs, got)
        torch.cuda.synchronize()
        assert lrkv.lrkv_query_static_scratch_status() == ("LRKV_OK", 0)
        assert torch.isfinite(got.float()).all()
        max_abs, rel = errors(to_np(got), to_np(ref))
        assert max_abs <= MAX_ABS and rel <= REL_L2, (seed, max_abs, rel)
        want = decode_oracle(q, k, v, u, b, offs, seq, mode, page_table=table)
        assert_parity(to_np(got), want, f"static scratch seed {seed}")


def test_static_scratch_reports_a_bad_page_id():
    q, k, v, u, b, offs, seq, table = _case(7, S=2, N=2, Hq=4, Hkv=2, L=1024, paged=True)
    S, N, Hq, d = q.shape
    prob = lrkv.make_problem(S, N, Hq, k.shape[1], d, u.shape[-1], lrkv.BASE_SHARED)
    bad = table.clone()
    bad[1, 3] = k.shape[0]  # one page id past the pool: that tile is skipped and flagged
    out = torch.empty_like(q)
    lrkv.lrkv_attn_decode_static_scratch(prob, q, lrkv.kv_view_paged(k, v, bad), seq, 1024, u, b, offs, out)
    st, flags = lrkv.lrkv_query_static_scratch_status(clear=False)
    assert st == "LRKV_ERR_DEVICE_FAULT" and flags & 0x4, (st, hex(flags))
    assert lrkv.lrkv_query_static_scratch_status()[0] == "LRKV_ERR_DEVICE_FAULT"  # read once more, then cleared
    assert lrkv.lrkv_query_static_scratch_status() == ("LRKV_OK", 0)
    # the next call clears the flags itself and, with a good table, raises none
    lrkv.lrkv_attn_decode_static_scratch(prob, q, lrkv.kv_view_paged(k, v, table), seq, 1024, u, b, offs, out)
    assert lrkv.lrkv_query_static_scratch_status() == ("LRKV_OK", 0)
    assert_parity(to_np(out), decode_oracle(q, k, v, u, b, offs, seq, lrkv.BASE_SHARED, page_table=table), "after")


def test_static_scratch_rejects_shapes_beyond_its_size():
    # 64 sessions x 8 KV heads x 16 rows over 4096 keys needs more partial records than the scratch holds
    prob = lrkv.make_problem(64, 8, 16, 8, 128, 16, lrkv.BASE_SHARED)
    need = lrkv.lrkv_decode_workspace_bytes(prob, 4096)
    assert need > (8 << 20)
    t = torch.zeros(16, dtype=torch.bfloat16, device=DEV)
    kv = lrkv.KVView(t.data_ptr(), t.data_ptr(), 8 * 4096 * 128, 4096 * 128, 128, None, 0, 0, 0, 0)
    uv = lrkv.UView(t.data_ptr(), 8 * 4096 * 16, 4096 * 16, 16, 4096)
    with pytest.raises(lrkv.LrkvError) as ei:
        lrkv.lrkv_attn_decode_static_scratch(prob, t, kv, t, 4096, uv, t, None, t)
    assert ei.value.name == "LRKV_ERR_WORKSPACE_TOO_SMALL"
