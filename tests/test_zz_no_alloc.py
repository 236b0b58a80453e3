"""Decode through the entry point that allocates nothing.

Some callers may not allocate device memory when they call attention: a
plug-in inside a serving engine whose device memory belongs to the engine's
own allocator, or a long-running server where cudaMalloc would synchronise the
device and can fail on a fragmented heap.  lrkv_attn_decode_static_scratch
serves them from one fixed scratch array inside the library.  These tests call
it through the C ABI, twice in a row (the scratch keeps the previous call's
contents), and compare with the regular entry point that takes a caller-owned
workspace, under the same tolerance as the other decode tests.
"""

import pytest
import torch

import lora_shared_kv_b200 as lrkv
from gpu_util import MAX_ABS, REL_L2, errors, to_np
from workloads.gen import _normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(seed, S=4, N=3, Hq=12, Hkv=2, d=128, r=16, L=2048):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = _normal((S, N, Hq, d), 1.0, g, DEV)
    k = _normal((S, Hkv, L, d), 1.0, g, DEV)
    v = _normal((S, Hkv, L, d), 1.0, g, DEV)
    u = _normal((S, N, L, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), 0.05, g, DEV)
    offs = torch.tensor([[100, 1500, 2047]] * S, dtype=torch.int32, device=DEV)
    seq = torch.tensor([L, L - 1, L // 2, 77][:S], dtype=torch.int32, device=DEV)
    return q, k, v, u, b, offs, seq


def test_static_scratch_decode_matches_workspace_decode_twice():
    for seed in (101, 202):  # two calls in a row on different inputs
        q, k, v, u, b, offs, seq = _case(seed)
        S, N, Hq, d = q.shape
        prob = lrkv.make_problem(S, N, Hq, k.shape[1], d, u.shape[-1], lrkv.BASE_SHARED)
        kv = lrkv.kv_view_dense(k, v)
        ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, k.shape[2]), dtype=torch.uint8, device=DEV)
        ref = torch.empty_like(q)
        lrkv.lrkv_attn_decode(prob, q, kv, seq, k.shape[2], u, b, offs, ref, ws)
        got = torch.full_like(q, float("nan"))
        lrkv.lrkv_attn_decode_static_scratch(prob, q, kv, seq, k.shape[2], u, b, offs, got)
        torch.cuda.synchronize()
        max_abs, rel = errors(to_np(got), to_np(ref))
        assert torch.isfinite(got.float()).all()
        assert max_abs <= MAX_ABS and rel <= REL_L2, (seed, max_abs, rel)


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
