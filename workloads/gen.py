"""Seeded random inputs.

Every tensor is drawn in fp32 from a seeded ``torch.Generator`` on the
requested device and rounded to bf16 (round-to-nearest-even, torch's cast).
The same tensors then feed both the CUDA path and, after a device-to-host
copy, the oracle.  Distributions (the reading where a workload leaves one
open): K, V, q and U ~ N(0, 1); B_i ~ N(0, b_std); A_i ~ N(0, 1/Dm) so that
X A_i ~ N(0, 1) like the stored U; offsets as the workload states.
"""

from dataclasses import dataclass
from typing import List, Optional

import torch

from .configs import BASE_SHARED, DecodeConfig, PrefillConfig

_CHUNK = 1 << 26


def seed_for(cfg) -> int:
    """Seed of a workload: 1000 * workload id + size index."""
    return 1000 * cfg.cfg_id + cfg.size_index


def _fill_normal_(out: torch.Tensor, std: float, gen: torch.Generator) -> torch.Tensor:
    flat = out.view(-1)
    n = flat.numel()
    for i in range(0, n, _CHUNK):
        m = min(_CHUNK, n - i)
        tmp = torch.randn(m, generator=gen, device=out.device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        flat[i:i + m].copy_(tmp)  # fp32 -> bf16 cast rounds to nearest even
    return out


def _normal(shape, std, gen, device, dtype=torch.bfloat16):
    return _fill_normal_(torch.empty(shape, dtype=dtype, device=device), std, gen)


@dataclass
class DecodeLayer:
    """One layer of decode inputs.

    q        [S, N, Hq, d] bf16
    k, v     dense: [S, Hkv, L, d] bf16;  paged: [P, Hkv, page, d] bf16 (physical pages)
    page_table  None (dense) or int32 [S, L/page] physical page of each logical page
    u        [S, N_U, L, r] bf16 (N_U = N in BaseShared, 1 in BaseLRShared)
    b        [N, r, Hkv*d] bf16
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    u: torch.Tensor
    b: torch.Tensor
    page_table: Optional[torch.Tensor] = None


@dataclass
class DecodeInputs:
    cfg: DecodeConfig
    layers: List[DecodeLayer]
    offsets: torch.Tensor     # int32 [S, N]
    seq_lens: torch.Tensor    # int32 [S]


def _draw_offsets(cfg: DecodeConfig, gen, device) -> torch.Tensor:
    if cfg.offset_range is not None:
        lo, hi = cfg.offset_range
        return torch.randint(lo, hi, (cfg.S, cfg.N), generator=gen, device=device,
                             dtype=torch.int64).to(torch.int32)
    offs = cfg.offsets if cfg.offsets is not None else (0,) * cfg.N
    assert len(offs) == cfg.N
    return torch.tensor(offs, dtype=torch.int32, device=device).repeat(cfg.S, 1).contiguous()


def make_decode_layer(cfg: DecodeConfig, gen: torch.Generator, device,
                      offsets: Optional[torch.Tensor] = None,
                      zero_before_offset: bool = False) -> DecodeLayer:
    S, N, Hq, Hkv, d, r, L = cfg.S, cfg.N, cfg.Hq, cfg.Hkv, cfg.d, cfg.r, cfg.L
    q = _normal((S, N, Hq, d), 1.0, gen, device)
    page_table = None
    if cfg.paged:
        assert L % cfg.page_size == 0
        n_lp = L // cfg.page_size
        n_pages = S * n_lp
        k = _normal((n_pages, Hkv, cfg.page_size, d), 1.0, gen, device)
        v = _normal((n_pages, Hkv, cfg.page_size, d), 1.0, gen, device)
        perm = torch.randperm(n_pages, generator=gen, device=device)
        page_table = perm.to(torch.int32).view(S, n_lp).contiguous()
    else:
        k = _normal((S, Hkv, L, d), 1.0, gen, device)
        v = _normal((S, Hkv, L, d), 1.0, gen, device)
    u = _normal((S, cfg.n_u, L, r), 1.0, gen, device)
    b = _normal((N, r, Hkv * d), cfg.b_std, gen, device)
    if zero_before_offset:
        assert offsets is not None
        offs = offsets.cpu()
        for s in range(S):
            for i in range(cfg.n_u):
                a = int(offs[s, i]) if cfg.mode == BASE_SHARED else int(offs[s].min())
                u[s, i, :a] = 0
    return DecodeLayer(q=q, k=k, v=v, u=u, b=b, page_table=page_table)


def make_decode_inputs(cfg: DecodeConfig, device="cpu", layers: Optional[int] = None,
                       seed: Optional[int] = None,
                       zero_before_offset: Optional[bool] = None) -> DecodeInputs:
    """All layers of a decode workload (distinct buffers per layer)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed_for(cfg) if seed is None else seed)
    offsets = _draw_offsets(cfg, gen, device)
    if zero_before_offset is None:
        zero_before_offset = cfg.cfg_id == 1  # the tiny case states zeroed rows
    n_layers = cfg.layers if layers is None else layers
    lays = [make_decode_layer(cfg, gen, device, offsets, zero_before_offset)
            for _ in range(n_layers)]
    seq_lens = torch.full((cfg.S,), cfg.L, dtype=torch.int32, device=device)
    return DecodeInputs(cfg=cfg, layers=lays, offsets=offsets, seq_lens=seq_lens)


def poison_lr_cache_(u: torch.Tensor, offsets: torch.Tensor, seq_lens: torch.Tensor,
                     mode: int) -> torch.Tensor:
    """Write NaN into every U row that no agent may read.

    u [S, N_U, Lcap, r]; rows t < a_i (BaseShared, per agent) or
    t < min_i a_i (BaseLRShared, shared U), and rows t >= seq_len, become NaN.
    A kernel that multiplies such rows by a zero weight instead of leaving them
    out produces NaN.
    """
    offs = offsets.cpu()
    sl = seq_lens.cpu()
    S, NU, Lcap, _ = u.shape
    for s in range(S):
        for i in range(NU):
            a = int(offs[s, i]) if mode == BASE_SHARED else int(offs[s].min())
            a = max(0, min(a, Lcap))
            u[s, i, :a] = float("nan")
            u[s, i, int(sl[s]):] = float("nan")
    return u


@dataclass
class PrefillInputs:
    """One layer, one session of a prefill chunk.

    q      [N, T, Hq, d]        queries of the new rows, one set per agent
    k, v   [1, Hkv, L0+T, d]    shared base cache, chunk rows [L0, L0+T) included
    u      [1, N_U, L0+T, r]    prefix rows [0, L0) drawn; chunk rows left NaN
                                 (the append fills them)
    x      [T, Dm]              hidden states of the chunk (shared by all agents)
    a_down [N_U, Dm, r]         LoRA down-projections A_i (one shared A in BaseLRShared)
    b      [N, r, Hkv*d]        LoRA up-projections B_i
    offsets int32 [N]
    """
    cfg: PrefillConfig
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    u: torch.Tensor
    x: torch.Tensor
    a_down: torch.Tensor
    b: torch.Tensor
    offsets: torch.Tensor


def make_prefill_inputs(cfg: PrefillConfig, device="cpu", seed: Optional[int] = None,
                        offsets=None) -> PrefillInputs:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed_for(cfg) if seed is None else seed)
    N, T, Hq, Hkv, d, r, L0, Dm = cfg.N, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.r, cfg.L0, cfg.Dm
    Ltot = L0 + T
    q = _normal((N, T, Hq, d), 1.0, gen, device)
    k = _normal((1, Hkv, Ltot, d), 1.0, gen, device)
    v = _normal((1, Hkv, Ltot, d), 1.0, gen, device)
    u = torch.full((1, cfg.n_u, Ltot, r), float("nan"), dtype=torch.bfloat16, device=device)
    if L0 > 0:
        u[:, :, :L0].copy_(_normal((1, cfg.n_u, L0, r), 1.0, gen, device))
    x = _normal((T, Dm), 1.0, gen, device)
    a_down = _normal((cfg.n_u, Dm, r), Dm ** -0.5, gen, device)
    b = _normal((N, r, Hkv * d), cfg.b_std, gen, device)
    if offsets is None:
        offs = cfg.offsets if cfg.offsets is not None else (0,) * N
        offsets = torch.tensor(offs, dtype=torch.int32, device=device)
    return PrefillInputs(cfg=cfg, q=q, k=k, v=v, u=u, x=x, a_down=a_down, b=b,
                         offsets=offsets.to(device=device, dtype=torch.int32))
