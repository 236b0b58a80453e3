"""Golden fixtures: the oracle's stored values, cross-checked by the brute force.

The fixtures under tests/golden/ were written by tests/golden/make_golden.py,
which calls only the oracle.  Here they are checked two ways: the 40-digit
brute force (independent code) must reproduce them, and the current oracle
must still give them (a regression guard on the oracle itself).
"""

import json
import os

import numpy as np

import oracle
from brute_decimal import brute_decode, brute_prefill

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(HERE, name)) as f:
        return json.load(f)


def test_golden_decode():
    fx = _load("tiny_decode.json")
    exp = np.array(fx["expected"])
    a = {k: np.array(fx[k]) for k in ("q", "k", "v", "u", "b", "offsets", "seq_lens")}
    got = oracle.decode(a["q"], a["k"], a["v"], a["u"], a["b"], a["offsets"], a["seq_lens"], fx["mode"])
    assert np.max(np.abs(got - exp)) <= 1e-15
    ref = np.array(brute_decode(fx["q"], fx["k"], fx["v"], fx["u"], fx["b"], fx["offsets"],
                                fx["seq_lens"], fx["mode"]))
    assert np.max(np.abs(ref - exp)) <= 1e-13


def test_golden_prefill():
    fx = _load("tiny_prefill.json")
    exp = np.array(fx["expected"])
    a = {k: np.array(fx[k]) for k in ("q", "k", "v", "u", "b", "offsets")}
    got = oracle.prefill_chunk(a["q"], a["k"], a["v"], a["u"], a["b"], a["offsets"], fx["ctx_len"], fx["mode"])
    assert np.max(np.abs(got - exp)) <= 1e-15
    ref = np.array(brute_prefill(fx["q"], fx["k"], fx["v"], fx["u"], fx["b"], fx["offsets"],
                                 fx["ctx_len"], fx["mode"]))
    assert np.max(np.abs(ref - exp)) <= 1e-13
