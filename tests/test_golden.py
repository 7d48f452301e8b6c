"""The C oracle reproduces the stored golden cases (written by
tests/golden/make_golden.py from the decimal brute force; each case cites
the passage whose semantics it fixes)."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "semantics_cases.json")


def _cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_oracle_reproduces_golden_case(case):
    assert case["cite"]
    q = np.array(case["q"], dtype=np.float64).astype(np.float32)
    k = np.array(case["k"], dtype=np.float64).astype(np.float32)
    v = np.array(case["v"], dtype=np.float64).astype(np.float32)
    got = oracle.attention(q, k, v, case["pos"], window=case["window"], scale=case["scale"],
                           n_kv_heads=case.get("n_kv_heads", 1))
    want = np.array([[[float(x) for x in row] for row in head] for head in case["expected"]])
    assert got.shape == want.shape
    for g, w in zip(got.ravel(), want.ravel()):
        if math.isnan(w):
            assert math.isnan(g)
        else:
            assert abs(g - w) <= 1e-12


def test_stored_cases_are_what_the_committed_script_writes():
    # the fixture is the brute force's output for the script's inputs, and
    # nothing else (no value in it came from anywhere but oracle.brute)
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_golden", os.path.join(os.path.dirname(__file__), "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    assert json.loads(json.dumps(mg.cases())) == _cases()
