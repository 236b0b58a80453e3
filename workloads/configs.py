"""Workload shapes.

Notation: S sessions, N agents (LoRA roles), Hq / Hkv query / KV heads,
G = Hq / Hkv, d head_dim, r LoRA rank, L cached context length, Dm hidden size.
Mode 0 is BaseShared (one low-rank cache U_i per agent), mode 1 is
BaseLRShared (one shared down-projection A, so one U shared by all agents);
both are the two sharing schemes of "LRAgent: Efficient KV Cache Sharing for
Multi-LoRA LLM Agents" (the review's reading, Fig. 2-3).
"""

from dataclasses import dataclass, field
from typing import Optional, Tuple

BASE_SHARED = 0
BASE_LR_SHARED = 1


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    cfg_id: int
    layers: int
    S: int
    N: int
    Hq: int
    Hkv: int
    d: int
    r: int
    Dm: int
    L: int
    mode: int = BASE_SHARED
    # aLoRA activation offsets: a fixed tuple (one per agent, same for all
    # sessions), or None with offset_range set (drawn per (session, agent)).
    offsets: Optional[Tuple[int, ...]] = None
    offset_range: Optional[Tuple[int, int]] = None
    b_std: float = 0.02
    paged: bool = False
    page_size: int = 64
    size_index: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def rows_per_kv_head(self) -> int:
        return self.N * self.G

    @property
    def n_u(self) -> int:
        return self.N if self.mode == BASE_SHARED else 1

    @property
    def queries_per_step(self) -> int:
        return self.S * self.N

    def kv_bytes_per_layer(self) -> int:
        return 2 * self.S * self.Hkv * self.L * self.d * 2


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    cfg_id: int
    N: int
    Hq: int
    Hkv: int
    d: int
    r: int
    Dm: int
    L0: int
    T: int
    mode: int = BASE_SHARED
    offsets: Optional[Tuple[int, ...]] = None
    b_std: float = 0.02
    size_index: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_u(self) -> int:
        return self.N if self.mode == BASE_SHARED else 1


# Tiny correctness case, one layer, Qwen-free toy shape.
CFG1 = DecodeConfig(name="tiny-decode-L256", cfg_id=1, layers=1, S=1, N=2, Hq=2, Hkv=1,
                    d=64, r=8, Dm=128, L=256, mode=BASE_SHARED, offsets=(128, 192),
                    b_std=0.05)
# Qwen2.5-Coder-1.5B-shaped decode (28 layers, GQA 12/2, d=128, Dm=1536),
# three roles at r=16, 32 sessions, 8192 shared tokens.
CFG2 = DecodeConfig(name="qwen2.5-coder-1.5b-decode-L8192-S32-N3", cfg_id=2, layers=28,
                    S=32, N=3, Hq=12, Hkv=2, d=128, r=16, Dm=1536, L=8192,
                    mode=BASE_SHARED, offsets=(6000, 7000, 7800), b_std=0.02)


def _cfg3(L: int, idx: int) -> DecodeConfig:
    # Qwen3-1.7B-shaped decode sweep, BaseLRShared (one U), two specialists.
    return DecodeConfig(name=f"qwen3-1.7b-lrshared-decode-L{L}-S16-N2", cfg_id=3, layers=28,
                        S=16, N=2, Hq=16, Hkv=8, d=128, r=16, Dm=2048, L=L,
                        mode=BASE_LR_SHARED, offsets=(0, 0), b_std=0.02, size_index=idx)


CFG3 = tuple(_cfg3(L, i) for i, L in enumerate((1024, 2048, 4096, 8192)))

# Long-context paged stress case: 8 agents, 65536 tokens in 64-token pages.
CFG5 = DecodeConfig(name="qwen3-1.7b-paged-decode-L65536-S4-N8", cfg_id=5, layers=28,
                    S=4, N=8, Hq=16, Hkv=8, d=128, r=16, Dm=2048, L=65536,
                    mode=BASE_SHARED, offset_range=(32768, 65536), b_std=0.02,
                    paged=True, page_size=64)

# Prefill chunk: 4 agents append 512 tokens onto a 16384-token shared cache.
CFG4 = PrefillConfig(name="qwen3-1.7b-prefill-L0-16384-T512-N4", cfg_id=4, N=4, Hq=16,
                     Hkv=8, d=128, r=32, Dm=2048, L0=16384, T=512, mode=BASE_SHARED,
                     offsets=(0, 0, 0, 0), b_std=0.02)

CONFIGS = {
    "cfg1": CFG1,
    "cfg2": CFG2,
    "cfg3_1k": CFG3[0],
    "cfg3_2k": CFG3[1],
    "cfg3_4k": CFG3[2],
    "cfg3_8k": CFG3[3],
    "cfg4": CFG4,
    "cfg5": CFG5,
}


def decode_config(key: str) -> DecodeConfig:
    c = CONFIGS[key]
    assert isinstance(c, DecodeConfig), key
    return c


def prefill_config(key: str) -> PrefillConfig:
    c = CONFIGS[key]
    assert isinstance(c, PrefillConfig), key
    return c
