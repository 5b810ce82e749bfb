"""The oracle against hand-derived closed-form cases stored in tests/golden/
(each case cites the passage whose definition it follows)."""
import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = json.load(open(os.path.join(HERE, "golden", "closed_forms.json")))["cases"]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_oracle_matches_hand_derived_case(case):
    q, k, v = (np.array(case[n], dtype=np.float64) for n in ("q", "k", "v"))
    window = None if case["window"] is None else tuple(case["window"])
    o, lse, _ = oracle.fwd(q, k, v, case["cu"], case["causal"], case["scale"], window=window)
    np.testing.assert_allclose(o, np.array(case["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(case["lse"]), rtol=0, atol=1e-12)


BWD_CASES = json.load(open(os.path.join(HERE, "golden", "closed_forms.json")))["backward_cases"]


@pytest.mark.parametrize("case", BWD_CASES, ids=[c["name"] for c in BWD_CASES])
def test_oracle_backward_matches_hand_derived_case(case):
    q, k, v, do = (np.array(case[n], dtype=np.float64) for n in ("q", "k", "v", "dout"))
    dq, dk, dv = oracle.bwd(q, k, v, do, case["cu"], case["causal"], case["scale"])
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        np.testing.assert_allclose(got, np.array(case[name]), rtol=0, atol=1e-12)
