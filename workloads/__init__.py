"""Seeded synthetic inputs for split-value-cache attention.

This module is shared by the oracle side (tests, CPU baseline) and the CUDA
side (tests, bench).  It holds only workload shapes and random draws: none of
the attention arithmetic lives here.

Shapes follow the models the pages name (Qwen2.5-Coder-1.5B on the RoleKV
page, "How we built it"; Qwen3-1.7B on the reuse-study page, section 2) and the
five workload descriptions of the hot path.  The pages' own evaluation data
(HotpotQA, ScienceQA, GSM8K, MBPP) is not used: N(0, 1) draws of the same
shapes stand in for it.
"""

from .configs import (  # noqa: F401
    DecodeConfig,
    PrefillConfig,
    CONFIGS,
    decode_config,
    prefill_config,
)
from .gen import (  # noqa: F401
    DecodeInputs,
    PrefillInputs,
    make_decode_inputs,
    make_prefill_inputs,
    make_decode_layer,
    poison_lr_cache_,
    seed_for,
)
