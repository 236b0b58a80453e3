"""Decode parity: the CUDA path (through the C ABI) against the fp64 oracle.

Sizes here finish in the oracle within seconds yet span several key tiles,
several CTAs per work item (the split merge), a ragged last tile, row groups,
both sharing modes, both head dims and all ranks.  Full-size workloads are in
test_gpu_fullsize.py.
"""

import zlib

import numpy as np
import pytest
import torch

from gpu_util import assert_parity, decode_gpu, decode_oracle, to_np
from workloads import CONFIGS, make_decode_inputs, poison_lr_cache_
from workloads.gen import _normal

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(seed, S, N, Hq, Hkv, d, r, Lcap, mode, offsets, seq_lens, paged=False, b_std=0.05):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = _normal((S, N, Hq, d), 1.0, g, DEV)
    k = _normal((S, Hkv, Lcap, d), 1.0, g, DEV)
    v = _normal((S, Hkv, Lcap, d), 1.0, g, DEV)
    nu = N if mode == 0 else 1
    u = _normal((S, nu, Lcap, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), b_std, g, DEV)
    offs = torch.tensor(offsets, dtype=torch.int32, device=DEV).reshape(S, N)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    return q, k, v, u, b, offs, sl


def test_tiny_config_with_poisoned_rows():
    cfg = CONFIGS["cfg1"]
    inp = make_decode_inputs(cfg, device=DEV)
    lay = inp.layers[0]
    u = lay.u.clone()
    poison_lr_cache_(u, inp.offsets, inp.seq_lens, cfg.mode)
    out = decode_gpu(lay.q, lay.k, lay.v, u, lay.b, inp.offsets, inp.seq_lens, cfg.L, cfg.mode)
    ref = decode_oracle(lay.q, lay.k, lay.v, lay.u, lay.b, inp.offsets, inp.seq_lens, cfg.mode)
    assert_parity(to_np(out), ref, "cfg1")


SHAPES = [
    # S, N, Hq, Hkv, d, r, Lcap, mode, offsets(S*N), seq_lens(S)
    (2, 3, 12, 2, 128, 16, 1000, 0, [0, 300, 999, 17, 64, 2000], [1000, 777]),
    (3, 2, 16, 8, 128, 16, 700, 1, [0, 100, 5, 5, 0, 0], [700, 1, 64]),
    (1, 5, 8, 1, 64, 32, 300, 0, [0, 10, 100, 200, 299], [300]),          # 40 rows: two row groups
    (2, 16, 4, 4, 128, 8, 130, 0, list(range(0, 160, 5))[:32], [130, 129]),  # 16 agents, G = 1
    (2, 2, 4, 2, 64, 8, 96, 1, [95, 3, 0, 0], [96, 65]),
    (1, 3, 12, 2, 128, 32, 4097, 0, [4000, 4096, 1], [4097]),
    (4, 2, 2, 1, 64, 16, 200, 0, [0, 0, 50, 300, 10, 10, 199, 0], [1, 0, 200, 63]),  # L=1, empty session
    # 17 to 24 rows per KV head (the key-split consumers): rank 8, shared U with
    # offsets inside a warp's 16 keys, an empty session
    (2, 3, 6, 1, 128, 8, 515, 1, [0, 250, 514, 3, 3, 0], [515, 0]),
    (3, 4, 5, 1, 64, 16, 450, 0, [0, 7, 449, 100, 1, 1, 1, 1, 64, 65, 200, 0], [450, 1, 449]),  # 20 rows
    (1, 3, 24, 3, 128, 16, 2000, 1, [0, 0, 0], [2000]),  # 24 rows, every offset 0: one Z pass
]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"S{s[0]}N{s[1]}Hq{s[2]}Hkv{s[3]}d{s[4]}r{s[5]}L{s[6]}m{s[7]}"
                                               for s in SHAPES])
def test_decode_shapes(shape):
    S, N, Hq, Hkv, d, r, Lcap, mode, offs, sls = shape
    q, k, v, u, b, o, sl = _case(zlib.crc32(str(shape).encode()) % 100000, S, N, Hq, Hkv, d, r, Lcap, mode, offs, sls)
    up = u.clone()
    poison_lr_cache_(up, o, sl, mode)
    kp, vp = k.clone(), v.clone()
    for s in range(S):
        kp[s, :, int(sl[s]):] = float("nan")
        vp[s, :, int(sl[s]):] = float("nan")
    out = decode_gpu(q, kp, vp, up, b, o, sl, Lcap, mode)
    ref = decode_oracle(q, k, v, u, b, o, sl, mode)
    res = to_np(out)
    for s in range(S):
        if int(sl[s]) == 0:
            assert np.all(res[s] == 0)
            ref[s] = 0.0
    assert_parity(res, ref, str(shape))


def test_fp32_output_and_many_segments():
    # one (session, head) item over 8192 keys: 128 tiles spread over up to 128 CTAs
    q, k, v, u, b, o, sl = _case(7, 1, 3, 6, 1, 128, 16, 8192, 0, [6000, 7000, 7800], [8192])
    out32 = decode_gpu(q, k, v, u, b, o, sl, 8192, 0, out_dtype=torch.float32)
    ref = decode_oracle(q, k, v, u, b, o, sl, 0)
    assert_parity(to_np(out32), ref, "fp32 out")
    out16 = decode_gpu(q, k, v, u, b, o, sl, 8192, 0)
    assert torch.equal(out32.to(torch.bfloat16), out16)


def test_workspace_reuse_is_deterministic():
    q, k, v, u, b, o, sl = _case(11, 2, 3, 12, 2, 128, 16, 2048, 0, [100, 1500, 2047, 0, 0, 0], [2048, 1999])
    from gpu_util import lrkv
    prob = lrkv.make_problem(2, 3, 12, 2, 128, 16, 0)
    ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, 2048), dtype=torch.uint8, device=DEV)
    a = decode_gpu(q, k, v, u, b, o, sl, 2048, 0, workspace=ws)
    c = decode_gpu(q, k, v, u, b, o, sl, 2048, 0, workspace=ws)
    assert torch.equal(a, c)


def test_offsets_null_means_zero():
    q, k, v, u, b, o, sl = _case(13, 2, 2, 4, 2, 128, 16, 333, 0, [0, 0, 0, 0], [333, 200])
    a = decode_gpu(q, k, v, u, b, None, sl, 333, 0)
    c = decode_gpu(q, k, v, u, b, o, sl, 333, 0)
    assert torch.equal(a, c)


def test_paged_equals_dense_bitwise():
    S, N, Hq, Hkv, d, r, page, n_lp = 3, 4, 8, 4, 128, 16, 64, 9
    L = page * n_lp
    offs = [0, 100, 576, 200, 64, 65, 300, 1, 500, 0, 0, 0]
    sls = [576, 500, 33]
    q, k, v, u, b, o, sl = _case(17, S, N, Hq, Hkv, d, r, L, 0, offs, sls)
    g = torch.Generator(device="cpu")
    g.manual_seed(5)
    perm = torch.randperm(S * n_lp, generator=g)
    table = perm.view(S, n_lp).to(torch.int32)
    kp = torch.empty((S * n_lp, Hkv, page, d), dtype=torch.bfloat16, device=DEV)
    vp = torch.empty_like(kp)
    for s in range(S):
        for lp in range(n_lp):
            kp[table[s, lp]] = k[s, :, lp * page:(lp + 1) * page]
            vp[table[s, lp]] = v[s, :, lp * page:(lp + 1) * page]
    dense = decode_gpu(q, k, v, u, b, o, sl, L, 0)
    paged = decode_gpu(q, kp, vp, u, b, o, sl, L, 0, page_table=table.to(DEV))
    assert torch.equal(dense, paged)
    ref = decode_oracle(q, k, v, u, b, o, sl, 0)
    assert_parity(to_np(paged), ref, "paged")


def test_shared_a_mode_equals_replicated_u():
    S, N = 2, 3
    q, k, v, u1, b, o, sl = _case(19, S, N, 12, 2, 128, 16, 900, 1, [0, 50, 400, 3, 3, 3], [900, 450])
    shared = decode_gpu(q, k, v, u1, b, o, sl, 900, 1)
    rep = u1.expand(S, N, 900, 16).contiguous()
    per_agent = decode_gpu(q, k, v, rep, b, o, sl, 900, 0)
    assert torch.equal(shared, per_agent)


def test_b_zero_is_base_attention_for_every_agent():
    q, k, v, u, b, o, sl = _case(23, 1, 3, 3, 1, 128, 16, 500, 0, [0, 10, 100], [500])
    q[:, 1:] = q[:, :1]           # same query for every agent
    out = decode_gpu(q, k, v, u, torch.zeros_like(b), o, sl, 500, 0)
    assert torch.equal(out[:, 0], out[:, 1]) and torch.equal(out[:, 0], out[:, 2])


def test_device_flags_are_raised_not_faulted():
    from gpu_util import lrkv
    q, k, v, u, b, o, sl = _case(29, 2, 2, 4, 2, 128, 16, 256, 0, [0, -5, 3, 3], [256, 999])
    prob = lrkv.make_problem(2, 2, 4, 2, 128, 16, 0)
    ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, 256), dtype=torch.uint8, device=DEV)
    decode_gpu(q, k, v, u, b, o, sl, 256, 0, workspace=ws, check_flags=False)
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_ERR_DEVICE_FAULT" and flags & 0x1 and flags & 0x2
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_OK" and flags == 0
    # a page id out of range is skipped and flagged
    table = torch.tensor([[0, 1, 2, 3], [4, 5, 6, 1000]], dtype=torch.int32, device=DEV)
    kp = k.view(2, 2, 4, 64, 128).permute(0, 2, 1, 3, 4).reshape(8, 2, 64, 128).contiguous()
    vp = v.view(2, 2, 4, 64, 128).permute(0, 2, 1, 3, 4).reshape(8, 2, 64, 128).contiguous()
    sl2 = torch.tensor([256, 256], dtype=torch.int32, device=DEV)
    decode_gpu(q, kp, vp, u, b, o.clamp(min=0), sl2, 256, 0, page_table=table, workspace=ws, check_flags=False)
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_ERR_DEVICE_FAULT" and flags & 0x4
