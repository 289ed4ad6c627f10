"""The oracle must keep reproducing its stored regression values
(tests/golden/oracle_regression.json, written by tests/golden/make_fixtures.py
from the oracle alone)."""
import json
import os

import numpy as np

from workloads import make_workload

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_stored_regression_values(oracle_mod):
    data = json.load(open(os.path.join(HERE, "golden", "oracle_regression.json")))
    assert len(data["cases"]) == 3
    for case in data["cases"]:
        w = make_workload(case["workload"], **case["overrides"])
        r = oracle_mod.forward_workload(w)
        for key in ("Y", "Z", "Qx"):
            if key in case:
                got = np.asarray(r[key])[..., :3, :4].reshape(-1)
                np.testing.assert_allclose(got, case[key], rtol=1e-12, atol=1e-15, err_msg=f"{case['workload']} {key}")
        if "Out" in case:
            got = np.asarray(r["Out"])[:, :3, :4].reshape(-1)
            np.testing.assert_allclose(got, case["Out"], rtol=1e-12, atol=1e-15)


def test_oracle_reproduces_hand_worked_example(oracle_mod):
    case = json.load(open(os.path.join(HERE, "golden", "hand_worked_flare.json")))
    out = oracle_mod.flare_forward(np.array(case["K"]), np.array(case["V"]), np.array(case["Q"]), None,
                                   case["scale"])
    np.testing.assert_allclose(out["Z"], case["Z"], rtol=1e-14)
    np.testing.assert_allclose(out["Y"], case["Y"], rtol=1e-14)


def test_oracle_gradients_match_stored_regression_values(oracle_mod):
    from workloads import make_upstream_grad
    data = json.load(open(os.path.join(HERE, "golden", "oracle_grad_regression.json")))
    assert len(data["cases"]) == 3
    for case in data["cases"]:
        w = make_workload(case["workload"], **case["overrides"])
        r = oracle_mod.backward_workload(w, make_upstream_grad(w))
        for key, want in case.items():
            if key in ("workload", "overrides"):
                continue
            got = np.asarray(r[key]).reshape(-1)[:48]
            np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-15, err_msg=f"{case['workload']} {key}")


def test_oracle_reproduces_hand_worked_gradient(oracle_mod):
    """Two tokens, one latent, D = 1: the gradients worked out by hand in
    tests/golden/hand_worked_flare_grad.json (derivation stored with them)."""
    case = json.load(open(os.path.join(HERE, "golden", "hand_worked_flare_grad.json")))
    g = oracle_mod.flare_backward(np.array(case["K"]), np.array(case["V"]), np.array(case["Q"]),
                                  np.array(case["dY"]), None, case["scale"])
    for k in ("dK", "dV", "dQ"):
        np.testing.assert_allclose(g[k], case[k], rtol=1e-14, atol=1e-15, err_msg=k)
