"""Writes oracle_regression.json (forward outputs) and
oracle_grad_regression.json (gradients) of the fp64 oracle on small seeded
cases, so that a later change to the oracle's arithmetic shows up as a test
failure.  The FLARE/FLARE++ pages print no worked example, so these are
regression values of the oracle itself (its correctness is pinned by
tests/test_oracle_pins.py), not values from the pages.

Run from the repository root:  python tests/golden/make_fixtures.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import bf16_bits_to_f64, make_upstream_grad, make_workload  # noqa: E402

CASES = [("flarepp_n1k", {"N": 96}), ("flare_n64k", {"N": 80, "B": 1, "M": 16}),
         ("flarepp_masked_n4k", {"N": 64, "B": 2, "M": 16})]


def sample(a):
    """A fixed, small selection of entries: first row block of every head."""
    a = np.asarray(a)
    return a[..., :3, :4].reshape(-1).tolist()


def main():
    oracle.build()
    out = {"note": "fp64 oracle regression values; see make_fixtures.py", "cases": []}
    for name, kw in CASES:
        w = make_workload(name, **kw)
        r = oracle.forward_workload(w)
        case = {"workload": name, "overrides": kw, "Y": sample(r["Y"]), "Z": sample(r["Z"])}
        if "Qx" in r:
            case["Qx"] = sample(r["Qx"])
        if "Out" in r:
            case["Out"] = np.asarray(r["Out"])[:, :3, :4].reshape(-1).tolist()
        out["cases"].append(case)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)

    grads = {"note": "fp64 oracle gradient regression values (dY from make_upstream_grad); see make_fixtures.py",
             "cases": []}
    for name, kw in CASES:
        w = make_workload(name, **kw)
        r = oracle.backward_workload(w, make_upstream_grad(w))
        keys = ("dK", "dV", "dQ") if w.variant == "flare" else ("dX", "dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0")
        grads["cases"].append({"workload": name, "overrides": kw,
                               **{k: np.asarray(r[k]).reshape(-1)[:48].tolist() for k in keys}})
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_grad_regression.json")
    with open(path, "w") as f:
        json.dump(grads, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
