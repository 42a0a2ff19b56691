"""Regression fixture of the oracle (stored by tests/golden/make_golden.py,
which calls only oracle/). A change to the oracle's arithmetic must show up
here and be justified by the passage it follows."""
import os

import numpy as np

from tests.golden import make_golden

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_stored_tiny_pair(oracle_mod):
    rows = [ln.split() for ln in open(os.path.join(HERE, "oracle_tiny_pair.txt")) if not ln.startswith("#")]
    assert len(rows) > 100
    outs = {layer["name"]: make_golden.compute(layer) for layer in make_golden.LAYERS}
    for name, i, h, e, val in rows:
        got = outs[name][int(i), int(h), int(e)]
        assert abs(got - float(val)) <= 1e-13 * max(1.0, abs(float(val))), (name, i, h, e)
