"""Regression pin: the oracle reproduces the stored tiny case (tests/golden/kda_tiny.json)."""
import json
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_reproduces_golden_tiny(oracle_lib):
    with open(os.path.join(HERE, "golden", "kda_tiny.json")) as f:
        d = json.load(f)
    arr = {k: np.array(v) for k, v in d.items() if k != "scale"}
    o, ht = oracle.kda_fwd(arr["q"], arr["k"], arr["v"], arr["g"], arr["beta"], d["scale"],
                           arr["h0"], lib=oracle_lib)
    np.testing.assert_allclose(o, arr["o"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(ht, arr["ht"], rtol=0, atol=1e-15)
    m = oracle.transition(arr["k"], arr["g"], arr["beta"], lib=oracle_lib)
    np.testing.assert_allclose(m, arr["m"], rtol=0, atol=1e-15)
