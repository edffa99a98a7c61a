"""Regression record of the oracle on the tiny fp32 workload (written by
tests/golden/make_golden.py from the oracle alone)."""
import json
import os

import numpy as np

from tests.golden.make_golden import compute

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_its_record():
    rec = json.load(open(os.path.join(HERE, "golden", "tiny_fp32_oracle.json")))
    now = compute()
    assert now["idx"] == rec["idx"]
    assert now["kept"] == rec["kept"]
    w = np.array([[float(v) for v in r] for r in rec["w"]])
    out = np.array([[float(v) for v in r] for r in rec["out"]])
    assert np.allclose(np.array([[float(v) for v in r] for r in now["w"]]), w, rtol=1e-13, atol=0)
    got = np.array([[float(v) for v in r] for r in now["out"]])
    assert np.max(np.abs(got - out)) <= 1e-12 * np.max(np.abs(out))
