"""The value projection into the split caches: [V_base | U_1..U_n] = X [W0_v | A_1..A_n]
through the C ABI, against the fp64 oracle.

Each output element is a bf16 rounding of an fp32 tensor-core sum, so it must
sit within bf16's unit roundoff (2^-8 relative: one rounding to the nearest of
8 significand bits) of the exact value, plus a small allowance for the fp32
accumulation.  Rows outside [start_row, start_row + T),
other sessions and the K cache stay untouched.  Token counts and Dm that are
not tile multiples, both sharing modes, a paged value cache, the K loop split
over clusters of 2 to 8 CTAs (few tiles; uneven K ranges; 128- and 256-column
tiles) and unsplit (many tiles) are covered."""

import numpy as np
import pytest
import torch

import lora_shared_kv_b200 as lrkv
import oracle
from gpu_util import to_np
from workloads.gen import _normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _close_bf16(got, ref):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    return bool(np.all(err <= np.abs(ref) * 2.0 ** -8 + 2e-4)), float(err.max())


@pytest.mark.parametrize("S,N,Hkv,d,r,mode,T,Dm,start,paged", [
    (2, 3, 2, 128, 16, 0, 200, 256, 5, False),
    (1, 4, 8, 128, 32, 0, 130, 2048, 0, False),
    (2, 2, 8, 128, 16, 1, 64, 200, 17, False),     # BaseLRShared: one U; Dm not a multiple of 64
    (1, 2, 2, 64, 8, 0, 300, 136, 64, False),
    (3, 3, 2, 128, 16, 0, 150, 512, 100, True),    # paged value cache
    (1, 4, 8, 128, 32, 0, 2100, 256, 3, False),    # enough tiles that the K loop is not split (256 columns)
    (1, 4, 8, 128, 32, 0, 1100, 256, 0, False),    # 256-column tiles with the K loop split
    (1, 2, 2, 64, 8, 0, 100, 1024, 0, False),      # one tile: K split over a cluster of 8
    (2, 3, 1, 128, 16, 1, 77, 136, 9, True),       # K split 3 ways, ragged last K step, paged
])
def test_value_projection_matches_oracle(S, N, Hkv, d, r, mode, T, Dm, start, paged):
    g = torch.Generator(device=DEV)
    g.manual_seed(T * 13 + Dm + start)
    n_u = N if mode == 0 else 1
    ncols = Hkv * d + n_u * r
    x = _normal((T, Dm), 1.0, g, DEV)
    w = _normal((Dm, ncols), Dm ** -0.5, g, DEV)
    L = start + T + 40
    session = S - 1
    prob = lrkv.make_problem(S, N, 2 * Hkv, Hkv, d, r, mode)
    u = torch.full((S, n_u, L, r), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    if not paged:
        k = torch.full((S, Hkv, L, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        v = torch.full_like(k, float("nan"))
        kv = lrkv.kv_view_dense(k, v)
    else:
        page = 64
        n_lp = (L + page - 1) // page
        n_pages = S * n_lp + 3
        k = torch.full((n_pages, Hkv, page, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        v = torch.full_like(k, float("nan"))
        gcpu = torch.Generator(device="cpu")
        gcpu.manual_seed(7)
        table = torch.randperm(n_pages, generator=gcpu)[:S * n_lp].view(S, n_lp).to(torch.int32).to(DEV)
        kv = lrkv.kv_view_paged(k, v, table)
    v_before, u_before, k_before = v.clone(), u.clone(), k.clone()
    lrkv.lrkv_value_projection(prob, x, w, kv, L, u, session, start, ws)
    torch.cuda.synchronize()
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_OK", (st, hex(flags))
    v_ref, u_ref = oracle.value_projection(x.cpu(), w.cpu(), Hkv, d, n_u, r)   # [Hkv, T, d], [n_u, T, r]
    if not paged:
        v_rows = v[session, :, start:start + T]
    else:
        pos = torch.arange(start, start + T, device=DEV)
        pg = table[session].long()[pos // 64]
        v_rows = v[pg, :, pos % 64].permute(1, 0, 2)                          # [Hkv, T, d]
    ok, err = _close_bf16(to_np(v_rows), v_ref)
    assert ok, ("V", err)
    ok, err = _close_bf16(to_np(u[session, :, start:start + T]), u_ref)
    assert ok, ("U", err)
    # nothing else written: other rows, other sessions, K
    assert torch.equal(k.view(torch.int16), k_before.view(torch.int16))
    u_mask = torch.ones_like(u, dtype=torch.bool)
    u_mask[session, :, start:start + T] = False
    assert torch.equal(u[u_mask].view(torch.int16), u_before[u_mask].view(torch.int16))
    v_mask = torch.ones_like(v, dtype=torch.bool)
    if not paged:
        v_mask[session, :, start:start + T] = False
    else:
        v_mask[pg, :, pos % 64] = False
    assert torch.equal(v[v_mask].view(torch.int16), v_before[v_mask].view(torch.int16))


@pytest.mark.parametrize("T,Dm,Hkv,d,n_u,r", [
    (512, 2048, 8, 128, 4, 32),   # the prefill workload's shape: 128-column tiles, K split over a cluster
    (1100, 256, 8, 128, 4, 32),   # 256-column tiles, K split
    (100, 1024, 2, 64, 2, 8),     # one column tile, split 8 ways
])
def test_value_projection_is_deterministic(T, Dm, Hkv, d, n_u, r):
    # the split K loop's partial tiles are summed in cluster-rank order, so repeated
    # calls give the same bits whatever order the CTAs finish in
    g = torch.Generator(device=DEV)
    g.manual_seed(T + Dm)
    ncols = Hkv * d + n_u * r
    x = _normal((T, Dm), 1.0, g, DEV)
    w = _normal((Dm, ncols), Dm ** -0.5, g, DEV)
    prob = lrkv.make_problem(1, n_u, 2 * Hkv, Hkv, d, r, 0)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    outs = []
    for _ in range(3):
        k = torch.zeros((1, Hkv, T, d), dtype=torch.bfloat16, device=DEV)
        v = torch.zeros_like(k)
        u = torch.zeros((1, n_u, T, r), dtype=torch.bfloat16, device=DEV)
        lrkv.lrkv_value_projection(prob, x, w, lrkv.kv_view_dense(k, v), T, u, 0, 0, ws)
        outs.append((v, u))
    torch.cuda.synchronize()
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_OK", (st, hex(flags))
    for v, u in outs[1:]:
        assert torch.equal(v.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(u.view(torch.int16), outs[0][1].view(torch.int16))
