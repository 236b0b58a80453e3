"""Write the tiny golden fixtures of this folder.

The pages print no worked numeric example, so these fixtures are the oracle's
own values on tiny bf16 inputs, written here by a script that calls only the
oracle.  The inputs are stored in the fixture (as float64 values that are exact
bf16 numbers), so the fixture does not depend on any random generator.
``tests/test_golden.py`` checks them against the 40-digit brute force, which
shares no code with the oracle, and against the current oracle.

Run from the repository root:  python tests/golden/make_golden.py
"""

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def _bf16(x):
    b = oracle.f32_to_bf16_bits_rne(np.asarray(x, dtype=np.float32))
    return oracle.bf16_bits_to_f64(b)


def main():
    g = np.random.default_rng(20260)
    S, N, Hq, Hkv, d, L, r = 1, 3, 4, 2, 8, 7, 2
    dec = dict(
        q=_bf16(g.standard_normal((S, N, Hq, d))),
        k=_bf16(g.standard_normal((S, Hkv, L, d))),
        v=_bf16(g.standard_normal((S, Hkv, L, d))),
        u=_bf16(g.standard_normal((S, N, L, r))),
        b=_bf16(g.standard_normal((N, r, Hkv * d)) * 0.3),
        offsets=np.array([[0, 3, 7]]),
        seq_lens=np.array([L]),
        mode=0,
    )
    out = oracle.decode(dec["q"], dec["k"], dec["v"], dec["u"], dec["b"], dec["offsets"],
                        dec["seq_lens"], 0)
    fix = {k: (v.tolist() if isinstance(v, np.ndarray) else v) for k, v in dec.items()}
    fix["expected"] = out.tolist()
    fix["source"] = ("oracle.decode on the stored inputs (BaseShared, offsets inside, at and past "
                     "the context); written by tests/golden/make_golden.py")
    with open(os.path.join(HERE, "tiny_decode.json"), "w") as f:
        json.dump(fix, f, indent=None)

    N2, T, L0 = 2, 3, 4
    pre = dict(
        q=_bf16(g.standard_normal((N2, T, Hq, d))),
        k=_bf16(g.standard_normal((Hkv, L0 + T, d))),
        v=_bf16(g.standard_normal((Hkv, L0 + T, d))),
        u=_bf16(g.standard_normal((1, L0 + T, r))),
        b=_bf16(g.standard_normal((N2, r, Hkv * d)) * 0.3),
        offsets=np.array([2, 5]),
        ctx_len=L0,
        mode=1,
    )
    out = oracle.prefill_chunk(pre["q"], pre["k"], pre["v"], pre["u"], pre["b"], pre["offsets"],
                               pre["ctx_len"], 1)
    fix = {k: (v.tolist() if isinstance(v, np.ndarray) else v) for k, v in pre.items()}
    fix["expected"] = out.tolist()
    fix["source"] = ("oracle.prefill_chunk on the stored inputs (BaseLRShared, causal chunk of 3 rows "
                     "after 4 context rows); written by tests/golden/make_golden.py")
    with open(os.path.join(HERE, "tiny_prefill.json"), "w") as f:
        json.dump(fix, f, indent=None)


if __name__ == "__main__":
    main()
