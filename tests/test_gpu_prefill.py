"""Prefill-chunk parity: the tcgen05 path (through the C ABI) against the fp64 oracle.

Row j of the chunk sits at absolute position L0 + j and sees keys t <= L0 + j.
The small cases span several 128-key blocks, a ragged last tile and block,
G in {1, 2, 3, 4, 5, 6, 7} (tiles of floor(128 / G) tokens when G does not
divide 128), both head dims, every rank, both sharing modes, offsets inside a
block, inside the chunk and before it; NaN-poisoned U rows must not leak.  The
full-size cases are the prefill workload (4 agents, 512 rows onto 16384) with
the low-rank append in front, checked on sampled rows, once with the
workload's offsets and once with offsets inside the context and the chunk.
"""

import zlib

import numpy as np
import pytest
import torch

import lora_shared_kv_b200 as lrkv
import oracle
from gpu_util import assert_parity, to_np
from workloads import CONFIGS, make_prefill_inputs
from workloads.gen import _normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, N, T, Hq, Hkv, d, r, L0, mode, offsets, extra=37):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    Ltot = L0 + T
    q = _normal((N, T, Hq, d), 1.0, g, DEV)
    k = _normal((1, Hkv, Ltot + extra, d), 1.0, g, DEV)
    v = _normal((1, Hkv, Ltot + extra, d), 1.0, g, DEV)
    k[:, :, Ltot:] = float("nan")
    v[:, :, Ltot:] = float("nan")
    nu = N if mode == 0 else 1
    u = _normal((1, nu, Ltot + extra, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), 0.05, g, DEV)
    offs = torch.tensor(offsets, dtype=torch.int32, device=DEV)
    return q, k, v, u, b, offs


def _poison(u, offs, mode, Ltot):
    up = u.clone()
    o = offs.cpu().tolist()
    for i in range(up.shape[1]):
        a = o[i] if mode == 0 else min(o)
        up[0, i, :a] = float("nan")
        up[0, i, Ltot:] = float("nan")
    return up


def prefill_gpu(q, k, v, u, b, offs, L0, T, mode, session=0, kv=None, out_dtype=torch.bfloat16):
    N, _, Hq, d = q.shape
    Hkv = k.shape[1]
    r = u.shape[-1]
    prob = lrkv.make_problem(k.shape[0] if kv is None else 1, N, Hq, Hkv, d, r, mode)
    if kv is None:
        kv = lrkv.kv_view_dense(k, v)
    ws = torch.zeros(max(256, lrkv.lrkv_prefill_workspace_bytes(prob, L0, T)), dtype=torch.uint8, device=DEV)
    out = torch.full((N, T, Hq, d), float("nan"), dtype=out_dtype, device=DEV)
    lrkv.lrkv_attn_prefill_chunk(prob, q, kv, session, L0, T, u, b, offs, out, ws)
    torch.cuda.synchronize()
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_OK", (st, hex(flags))
    return out


SHAPES = [
    # N, T, Hq, Hkv, d, r, L0, mode, offsets
    (2, 100, 4, 2, 128, 32, 300, 0, [0, 150]),
    (3, 64, 8, 8, 128, 16, 0, 1, [0, 5, 40]),
    (1, 200, 4, 1, 64, 16, 1000, 0, [900]),
    (2, 130, 16, 8, 128, 32, 4096, 0, [4200, 0]),
    (2, 1, 8, 4, 128, 16, 77, 1, [30, 0]),
    (1, 257, 2, 2, 64, 32, 129, 0, [129]),
    # Qwen2.5-Coder-1.5B role switch (RoleKV): 12/2 heads (G = 6, tiles of 21 tokens = 126 rows),
    # a 64-row role header onto 8192 shared tokens, three roles, offsets inside the context and the chunk
    (3, 64, 12, 2, 128, 16, 8192, 0, [6000, 7000, 8200]),
    (2, 90, 10, 2, 64, 8, 500, 0, [0, 530]),       # G = 5, rank 8
    (2, 50, 6, 2, 128, 8, 300, 1, [10, 320]),      # G = 3, rank 8, one shared U
    (1, 30, 7, 1, 128, 32, 200, 0, [100]),         # G = 7
]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"N{s[0]}T{s[1]}Hq{s[2]}Hkv{s[3]}d{s[4]}r{s[5]}L{s[6]}m{s[7]}"
                                               for s in SHAPES])
def test_prefill_shapes(shape):
    N, T, Hq, Hkv, d, r, L0, mode, offs = shape
    q, k, v, u, b, o = _inputs(zlib.crc32(str(shape).encode()) % 100000, N, T, Hq, Hkv, d, r, L0, mode, offs)
    Ltot = L0 + T
    out = prefill_gpu(q, k, v, _poison(u, o, mode, Ltot), b, o, L0, T, mode)
    ref = oracle.prefill_chunk(q.cpu(), k[0, :, :Ltot].cpu(), v[0, :, :Ltot].cpu(), u[0, :, :Ltot].cpu(),
                               b.cpu(), o.cpu(), L0, mode)
    assert_parity(to_np(out), ref, str(shape))


def test_prefill_fp32_out_matches_bf16_rounding():
    q, k, v, u, b, o = _inputs(5, 2, 90, 4, 2, 128, 32, 500, 0, [0, 250])
    o32 = prefill_gpu(q, k, v, u, b, o, 500, 90, 0, out_dtype=torch.float32)
    o16 = prefill_gpu(q, k, v, u, b, o, 500, 90, 0)
    ref = oracle.prefill_chunk(q.cpu(), k[0, :, :590].cpu(), v[0, :, :590].cpu(), u[0, :, :590].cpu(), b.cpu(),
                               o.cpu(), 500, 0)
    assert_parity(to_np(o32), ref, "fp32")
    assert torch.equal(o32.to(torch.bfloat16), o16)


def test_prefill_paged_equals_dense_bitwise():
    N, T, Hq, Hkv, d, r, L0 = 2, 70, 4, 2, 128, 16, 250
    Ltot = L0 + T
    n_lp = (Ltot + 63) // 64
    q, k, v, u, b, o = _inputs(9, N, T, Hq, Hkv, d, r, L0, 0, [0, 100], extra=n_lp * 64 - Ltot)
    k[:, :, Ltot:] = 0
    v[:, :, Ltot:] = 0
    gcpu = torch.Generator(device="cpu")
    gcpu.manual_seed(3)
    n_pages = n_lp + 5
    perm = torch.randperm(n_pages, generator=gcpu)[:n_lp]
    kp = torch.zeros((n_pages, Hkv, 64, d), dtype=torch.bfloat16, device=DEV)
    vp = torch.zeros_like(kp)
    for lp in range(n_lp):
        kp[perm[lp]] = k[0, :, lp * 64:(lp + 1) * 64]
        vp[perm[lp]] = v[0, :, lp * 64:(lp + 1) * 64]
    table = perm.to(torch.int32).view(1, n_lp).to(DEV)
    dense = prefill_gpu(q, k, v, u, b, o, L0, T, 0)
    paged = prefill_gpu(q, kp, vp, u, b, o, L0, T, 0, kv=lrkv.kv_view_paged(kp, vp, table))
    assert torch.equal(dense, paged)


def test_prefill_rows_before_offset_equal_base():
    # offsets past the whole chunk: the adapter never switches on, so every agent gives the base output
    N, T, L0 = 3, 64, 200
    q, k, v, u, b, o = _inputs(13, N, T, 4, 2, 128, 32, L0, 0, [10 ** 6] * N)
    q[1:] = q[:1]
    out = prefill_gpu(q, k, v, u, b, o, L0, T, 0)
    assert torch.equal(out[0], out[1]) and torch.equal(out[0], out[2])
    base = prefill_gpu(q, k, v, u, torch.zeros_like(b), o, L0, T, 0)
    assert torch.equal(out, base)


@pytest.mark.parametrize("offsets,rows", [
    (None, [0, 1, 63, 64, 200, 383, 384, 511]),
    # aLoRA boundaries inside the 16384-token context and one inside the chunk (row 216):
    # rows on both sides of it
    ((9000, 12000, 16000, 16600), [0, 1, 64, 200, 215, 216, 217, 300, 511]),
], ids=["workload-offsets", "offsets-inside"])
def test_prefill_workload_with_append_sampled(offsets, rows):
    cfg = CONFIGS["cfg4"]
    offs = None if offsets is None else torch.tensor(offsets, dtype=torch.int32)
    inp = make_prefill_inputs(cfg, device=DEV, offsets=offs)
    lrkv.lrkv_append_lr_cache(inp.x, inp.a_down, inp.u, session=0, start_row=cfg.L0)
    out = prefill_gpu(inp.q, inp.k, inp.v, inp.u, inp.b, inp.offsets, cfg.L0, cfg.T, cfg.mode)
    ref = oracle.prefill_chunk(inp.q.cpu(), inp.k[0].cpu(), inp.v[0].cpu(), inp.u[0].cpu(), inp.b.cpu(),
                               inp.offsets.cpu(), cfg.L0, cfg.mode, rows=rows)
    got = to_np(out)
    assert_parity(got[:, rows], ref[:, rows], "prefill workload")
    assert torch.isfinite(out.float()).all()
    if offsets is not None:
        # rows whose every visible key lies before the last agent's offset carry no adapter term
        base = prefill_gpu(inp.q, inp.k, inp.v, inp.u, torch.zeros_like(inp.b), inp.offsets, cfg.L0, cfg.T,
                           cfg.mode)
        early = [j for j in rows if cfg.L0 + j < offsets[3]]
        assert early and torch.equal(out[3, early], base[3, early])
