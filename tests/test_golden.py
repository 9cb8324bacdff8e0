"""Golden fixtures: hand-derived record bytes, and a regression snapshot of the oracle."""
import json
import os

import numpy as np

from oracle import oracle as orc
from tests.helpers import bf16_bits

HERE = os.path.join(os.path.dirname(__file__), "golden")
D = 128


def _expand(spec):
    out = []
    for part in spec.split():
        body, _, rep = part.partition("*")
        vals = [int(x, 16) for x in body.split(",")]
        out += vals * (int(rep) if rep else 1)
    return out


def _cases():
    cases = {}
    for line in open(os.path.join(HERE, "pack_examples.txt")):
        if line.startswith("#") or not line.strip():
            continue
        name, field, spec = line.split(None, 2)
        cases.setdefault(name, {})[field] = _expand(spec)
    return cases


def test_hand_derived_records():
    d = np.arange(D)
    inputs = {"q2": (2, d % 4, -1 + 0.5 * ((d // 4) % 4)), "q4": (4, d % 16, d % 16)}
    for name, exp in _cases().items():
        bits, k, v = inputs[name]
        rec = orc.pack_record(bits, bf16_bits(k), bf16_bits(v))
        cb = D * bits // 8
        assert list(rec[:cb]) == exp["K"]
        assert list(rec[cb:2 * cb]) == exp["V"]
        assert list(rec[2 * cb:]) == exp["meta"]


def test_oracle_regression_snapshot():
    """The oracle's outputs on the 2k-token workload are unchanged since the snapshot
    (written by tests/golden/make_golden.py, which calls only the oracle)."""
    from tests.golden.make_golden import run_tiny
    snap = json.load(open(os.path.join(HERE, "tiny_b1_ctx2k.json")))
    got = run_tiny()
    assert got == snap
