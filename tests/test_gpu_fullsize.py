"""Full-size decode workloads, in the launch configuration the bench times.

Each workload is built and run by the bench's own runner (all layers, one
CUDA-graph replay); the oracle then checks sampled (layer, session) pairs
one by one, all agents and heads of each, at the full context length.
"""

import numpy as np
import pytest
import torch

from gpu_util import assert_parity, decode_oracle, to_np

pytestmark = pytest.mark.gpu

CASES = [
    ("cfg2", [0, 13, 27], [0, 31]),
    ("cfg3_1k", [0, 27], [0, 15]),
    ("cfg3_2k", [5], [3]),
    ("cfg3_4k", [9], [7]),
    ("cfg3_8k", [0, 27], [0, 15]),
    ("cfg5", [0, 27], [2]),
]


@pytest.mark.parametrize("key,layers,sessions", CASES, ids=[c[0] for c in CASES])
def test_fullsize_sampled(key, layers, sessions):
    import bench
    from workloads import CONFIGS
    cfg = CONFIGS[key]
    runner = bench.DecodeRunner(cfg, torch.device("cuda", 0))
    runner.capture()
    runner.step()
    torch.cuda.synchronize()
    st, flags = runner.lrkv.lrkv_query_device_status(runner.ws)
    assert st == "LRKV_OK", (st, hex(flags))
    inp = runner.inp
    for li in layers:
        lay = inp.layers[li]
        got = to_np(runner.outs[li])
        ref = decode_oracle(lay.q, lay.k, lay.v, lay.u, lay.b, inp.offsets, inp.seq_lens, cfg.mode,
                            page_table=lay.page_table, sessions=sessions)
        for s in sessions:
            assert_parity(got[s], ref[s], f"{key} layer {li} session {s}")
    # every output of every layer is finite
    for li in range(len(inp.layers)):
        assert torch.isfinite(runner.outs[li].float()).all(), f"{key} layer {li}"
    del runner
    torch.cuda.empty_cache()
