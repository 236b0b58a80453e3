"""The cache-sharing comparison that bench.py reports, checked against the fp64
oracle: the split value cache, per-agent private caches (non-shared) and the
base cache alone (full-shared), all through the same decode kernel.

- non-shared runs every agent as its own session over its own K and
  materialised V_i = V_base + Umask_i B_i with B = 0 ("LRAgent" review, Fig. 2:
  the Non-Shared baseline); it computes the same attention as the split cache,
  so it must match oracle.decode of the split problem (its only extra error is
  the bf16 rounding of V_i);
- full-shared drops the adapter's value term (same page, Fig. 2: FullShared,
  which shares the whole cache) and must match oracle.decode with B = 0;
- the shared arm must match oracle.decode of the split problem as well.
Sampled sessions of every layer the comparison times are checked element by
element under the stated tolerance."""

import dataclasses

import pytest
import torch

import bench
from gpu_util import assert_parity, decode_oracle, to_np
from workloads import CONFIGS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("key,over,sessions", [
    ("cfg2", dict(S=3, L=1000, layers=2), [0, 2]),                        # BaseShared, offsets inside the context
    ("cfg3_1k", dict(S=2, layers=2), [0, 1]),                             # BaseLRShared
    ("cfg5", dict(S=2, L=4096, layers=1, offset_range=(100, 4000)), [1]),  # paged, random offsets
])
def test_sharing_arms_match_the_oracle(key, over, sessions):
    cfg = dataclasses.replace(CONFIGS[key], **over)
    runner = bench.DecodeRunner(cfg, torch.device("cuda", 0))
    res, arms = bench.sharing_comparison(runner, steps=2, warmup=1, return_outputs=True)
    assert res["layers_timed"] == cfg.layers
    assert res["max_abs_non_shared_vs_shared"] <= 1e-2, res
    assert res["cache_bytes_per_layer_non_shared"] > res["cache_bytes_per_layer_shared"]
    assert res["ms_per_layer_non_shared"] > 0 and res["ms_per_layer_full_shared"] > 0
    inp = runner.inp
    for li in range(cfg.layers):
        lay = inp.layers[li]
        split = decode_oracle(lay.q, lay.k, lay.v, lay.u, lay.b, inp.offsets, inp.seq_lens, cfg.mode,
                              page_table=lay.page_table, sessions=sessions)
        base = decode_oracle(lay.q, lay.k, lay.v, lay.u, torch.zeros_like(lay.b), inp.offsets, inp.seq_lens,
                             cfg.mode, page_table=lay.page_table, sessions=sessions)
        shared, non_shared, full = (to_np(arms[a][li]) for a in ("shared", "non_shared", "full_shared"))
        for s in sessions:
            assert_parity(shared[s], split[s], f"{key} shared layer {li} session {s}")
            assert_parity(non_shared[s], split[s], f"{key} non-shared layer {li} session {s}")
            assert_parity(full[s], base[s], f"{key} full-shared layer {li} session {s}")
