"""The stored small problems of tests/golden/attn_small.json.

The file holds seeded inputs and the fp64 oracle's O, LSE, dQ, dK and dV for them
(written by tests/golden/make_golden.py).  Here, on the CPU: the stored inputs are
exactly what the seeded generator makes, the oracle still reproduces the stored
results (any change to its arithmetic shows), and the independent scalar brute
force agrees with the stored results too.
"""

import json
import os

import numpy as np
import pytest

import oracle
from oracle.brute import brute_bwd, brute_fwd
from exact_io_aware_74_b200.workloads import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "attn_small.json")


def _cases():
    with open(GOLDEN) as fh:
        return json.load(fh)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_golden_inputs_are_the_seeded_inputs(case):
    x = make_inputs(case["B"], case["H"], case["N"], case["d"], case["dtype"], seed=case["seed"],
                    with_do=True)
    for n in ("q", "k", "v", "do"):
        assert np.array_equal(x[n].double().numpy(), np.asarray(case[n]))


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_oracle_reproduces_golden(case):
    q, k, v, do = (np.asarray(case[n]) for n in ("q", "k", "v", "do"))
    o, lse = oracle.attn_fwd_ref(q, k, v, case["scale"], case["causal"])
    dq, dk, dv = oracle.attn_bwd_ref(q, k, v, do, case["scale"], case["causal"])
    for got, name in ((o, "o"), (lse, "lse"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        np.testing.assert_allclose(got, np.asarray(case[name]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_brute_force_agrees_with_golden(case):
    q, k, v, do = (np.asarray(case[n]) for n in ("q", "k", "v", "do"))
    bo, blse = brute_fwd(q, k, v, case["scale"], case["causal"])
    bq, bk, bv = brute_bwd(q, k, v, do, case["scale"], case["causal"])
    for got, name in ((bo, "o"), (blse, "lse"), (bq, "dq"), (bk, "dk"), (bv, "dv")):
        ref = np.asarray(case[name])
        assert np.max(np.abs(np.asarray(got) - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
