"""The oracle still reproduces its committed fingerprint (tests/golden/oracle_regression.json,
written by tests/golden/make_oracle_regression.py, which calls only the oracle). A failure
means the oracle's arithmetic changed: the change must name the passage that justifies it,
and the fingerprint is then rewritten by that script."""
import importlib.util
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _script():
    spec = importlib.util.spec_from_file_location("make_oracle_regression",
                                                  os.path.join(HERE, "golden", "make_oracle_regression.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_oracle_matches_its_committed_fingerprint():
    want = json.load(open(os.path.join(HERE, "golden", "oracle_regression.json")))
    got = _script().compute()
    for name in ("bf16_cache", "q8_cache"):
        assert got[name]["pos"] == want[name]["pos"]
        np.testing.assert_allclose(got[name]["S_l2"], want[name]["S_l2"], rtol=1e-9)
        for g, w in zip(got[name]["steps"], want[name]["steps"]):
            assert g["top_index"] == w["top_index"]
            np.testing.assert_allclose(g["top_value"], w["top_value"], rtol=1e-9, atol=1e-12)
            np.testing.assert_allclose([g["sum"], g["l2"]], [w["sum"], w["l2"]], rtol=1e-9, atol=1e-9)
    assert got["accept_sampled"]["n"] == want["accept_sampled"]["n"]
    assert got["accept_sampled"]["committed"] == want["accept_sampled"]["committed"]
