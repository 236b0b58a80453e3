"""Low-rank cache append: the CUDA path is bit-exact against the oracle's
fixed-order fp32 reference, and writes only the rows it is asked to."""

import numpy as np
import pytest
import torch

import lora_shared_kv_b200 as lrkv
import oracle
from workloads import CONFIGS, make_prefill_inputs
from workloads.gen import _normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits_t(t):
    return t.view(torch.int16)


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("T,Dm,r,n_a,start,cap", [
    (1, 128, 8, 2, 0, 256),
    (37, 1536, 16, 3, 100, 200),
    (512, 2048, 32, 4, 16384, 16896),
    (5, 65, 16, 1, 3, 8),
    (70, 100, 8, 2, 0, 100),
    (17, 300, 32, 1, 40, 64),
    # Dm a multiple of 8: the pipelined path, with a partial last k-chunk and token block
    (70, 200, 8, 2, 0, 100),
    (33, 136, 32, 3, 5, 64),
    (1, 8, 16, 1, 0, 4),
    (130, 1032, 16, 2, 7, 200),
])
def test_append_bit_exact(T, Dm, r, n_a, start, cap):
    g = torch.Generator(device=DEV)
    g.manual_seed(T * 7 + Dm)
    x = _normal((T, Dm), 1.0, g, DEV)
    a = _normal((n_a, Dm, r), Dm ** -0.5, g, DEV)
    S = 2
    u = torch.full((S, n_a, cap, r), float("nan"), dtype=torch.bfloat16, device=DEV)
    before = u.clone()
    lrkv.lrkv_append_lr_cache(x, a, u, session=1, start_row=start)
    torch.cuda.synchronize()
    want = oracle.ref_append_fp32(x.cpu(), a.cpu())              # [n_a, T, r] bits
    got = _bits(u[1, :, start:start + T])
    assert np.array_equal(got, want)
    # nothing else touched
    mask = torch.ones_like(u, dtype=torch.bool)
    mask[1, :, start:start + T] = False
    assert torch.equal(_nan_bits(u[mask]), _nan_bits(before[mask]))


def _nan_bits(t):
    return t.view(torch.int16)


def test_append_prefill_workload_rows():
    cfg = CONFIGS["cfg4"]
    inp = make_prefill_inputs(cfg, device=DEV)
    lrkv.lrkv_append_lr_cache(inp.x, inp.a_down, inp.u, session=0, start_row=cfg.L0)
    torch.cuda.synchronize()
    want = oracle.ref_append_fp32(inp.x.cpu(), inp.a_down.cpu())
    assert np.array_equal(_bits(inp.u[0, :, cfg.L0:]), want)


@pytest.mark.parametrize("Dm,r,ranges", [
    (2048, 32, [(0, 512), (100, 611), (300, 301), (50, 50)]),        # BaseShared catch-up, one empty range
    (1536, 16, [(7, 300), (0, 64), (129, 130)]),
    (200, 8, [(5, 77)]),                                              # BaseLRShared: one shared U
    (100, 16, [(3, 40), (0, 9)]),                                     # Dm not a multiple of 8: generic path
    (64, 8, [(i, i + 3 * i + 1) for i in range(18)]),                 # more agents than one launch takes
])
def test_append_ranges_bit_exact(Dm, r, ranges):
    n_a = len(ranges)
    x_rows = max(e for _, e in ranges) + 5
    g = torch.Generator(device=DEV)
    g.manual_seed(Dm * 31 + r + n_a)
    x = _normal((x_rows, Dm), 1.0, g, DEV)
    a = _normal((n_a, Dm, r), Dm ** -0.5, g, DEV)
    u = torch.full((2, n_a, x_rows + 3, r), float("nan"), dtype=torch.bfloat16, device=DEV)
    before = u.clone()
    lrkv.lrkv_append_lr_cache_ranges(x, a, u, session=1, row_begin=[b for b, _ in ranges],
                                     row_end=[e for _, e in ranges])
    torch.cuda.synchronize()
    for i, (b, e) in enumerate(ranges):
        if e > b:
            want = oracle.ref_append_fp32(x[b:e].cpu(), a[i:i + 1].cpu())[0]   # [e - b, r] bits
            assert np.array_equal(_bits(u[1, i, b:e]), want), (i, b, e)
        # nothing outside the range, and nothing in the other session
        outside = torch.ones(x_rows + 3, dtype=torch.bool)
        outside[b:e] = False
        assert torch.isnan(u[1, i, outside.to(DEV)].float()).all()
    assert torch.equal(_bits_t(u[0]), _bits_t(before[0]))
