"""The cache-sharing comparison that bench.py reports: the split value cache
against per-agent private caches (non-shared) and the base cache alone
(full-shared), all through the same decode kernel.

Non-shared runs every agent as its own session over its own K and materialised
V_i = V_base + Umask_i B_i with B = 0, so its outputs must agree with the shared
path's up to the bf16 rounding of V_i; full-shared drops the adapter term and
must equal the shared path with B = 0."""

import dataclasses

import pytest
import torch

import bench
from workloads import CONFIGS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("key,over", [
    ("cfg2", dict(S=3, L=1000, layers=2)),                       # BaseShared, offsets inside the context
    ("cfg3_1k", dict(S=2, layers=2)),                            # BaseLRShared
    ("cfg5", dict(S=2, L=4096, layers=1, offset_range=(100, 4000))),  # paged, random offsets
])
def test_sharing_comparison_agrees(key, over):
    cfg = dataclasses.replace(CONFIGS[key], **over)
    runner = bench.DecodeRunner(cfg, torch.device("cuda", 0))
    res = bench.sharing_comparison(runner, steps=2, warmup=1)
    assert res["layers_timed"] == cfg.layers
    assert res["max_abs_non_shared_vs_shared"] <= 1e-2, res
    assert res["cache_bytes_per_layer_non_shared"] > res["cache_bytes_per_layer_shared"]
    assert res["ms_per_layer_non_shared"] > 0 and res["ms_per_layer_full_shared"] > 0
