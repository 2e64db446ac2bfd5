"""GPU parity on the stored small problems of tests/golden/attn_small.json.

Ragged tiny shapes (N = 5 and 7 rows in one 128-row tile, head dims 8 and 16 in
64-wide tiles) through the C-ABI, against the stored fp64 results: O max-abs
2e-2 (bf16) / 5e-3 (fp16), LSE 1e-3, gradients 1e-2 x max|reference|.
"""

import json
import os

import numpy as np
import pytest
import torch

from exact_io_aware_74_b200 import fa2

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "attn_small.json")
O_TOL = {"bf16": 2e-2, "fp16": 5e-3}
DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def _cases():
    with open(GOLDEN) as fh:
        return json.load(fh)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_cuda_path_matches_golden(case):
    q, k, v, do = (torch.tensor(case[n], dtype=torch.float64).to(DT[case["dtype"]]).cuda()
                   for n in ("q", "k", "v", "do"))
    s, causal = case["scale"], case["causal"]
    o, lse = fa2.forward(q, k, v, s, causal)
    dq, dk, dv = fa2.backward(q, k, v, o, do, lse, s, causal)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    assert np.max(np.abs(o.cpu().double().numpy() - np.asarray(case["o"]))) <= O_TOL[case["dtype"]]
    assert np.max(np.abs(lse.cpu().double().numpy() - np.asarray(case["lse"]))) <= 1e-3
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        ref = np.asarray(case[name])
        assert np.max(np.abs(got.cpu().double().numpy() - ref)) <= 1e-2 * max(np.max(np.abs(ref)), 1e-3)
