"""The oracle against its stored regression record (tests/golden/oracle_small.json, written
by tests/golden/make_golden.py from oracle/ alone; the pages print no worked example, so
this is a change detector for the oracle, not a pin)."""
import importlib.util
import json
import os

import numpy as np

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_its_regression_record():
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    stored = json.load(open(os.path.join(HERE, "oracle_small.json")))
    assert "oracle/ only" in stored["about"]
    now = mg.compute()
    assert set(now) == set(stored["values"])
    for name, vals in stored["values"].items():
        assert np.allclose(np.asarray(now[name]), np.asarray(vals), rtol=1e-12, atol=1e-14), name
