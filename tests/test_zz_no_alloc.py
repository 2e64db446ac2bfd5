"""The allocation-free backward, fa2_bwd_noalloc, against the ordinary fa2_bwd.

fa2_bwd_noalloc is for callers that cannot call cudaMalloc (runtimes that hand out
device memory only from their own pool, latency-critical code that must not take
the synchronisation an allocation can cause): it runs the same kernels with the
library's fixed 32 MiB device buffer as scratch.  Two calls in a row, the second
on other inputs and a smaller problem, must both match fa2_bwd (with a
caller-provided workspace) within the backward tolerance, so a stale buffer from
the first call cannot leak into the second.

This file is collected last on purpose, and it also passes in a fresh process.
"""

import math

import pytest
import torch

from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

GRAD_REL = 1e-2  # the backward parity tolerance: max-abs error <= 1e-2 x max|reference|


def _close(got, ref):
    scale = max(float(ref.float().abs().max()), 1e-3)
    return float((got.float() - ref.float()).abs().max()) <= GRAD_REL * scale


def _case(name):
    """(inputs, scale, causal) of one backward problem."""
    if name == "workload_d64_causal":
        w = WORKLOADS["fwdbwd_bf16_b4h16_n1024_d64_causal"]
        return workload_inputs(w), w.scale, w.causal
    if name == "b2h4_n700_d128_causal":
        return make_inputs(2, 4, 700, 128, "bf16", seed=41, with_do=True), 1 / math.sqrt(128), True
    if name == "b1h3_n300_d128_causal":
        return make_inputs(1, 3, 300, 128, "bf16", seed=42, with_do=True), 1 / math.sqrt(128), True
    if name == "b2h8_n500_d64":
        return make_inputs(2, 8, 500, 64, "bf16", seed=43, with_do=True), 0.125, False
    raise KeyError(name)


def _noalloc_matches_backward(name):
    x, scale, causal = _case(name)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, scale, causal)
    ref = fa2.backward(q, k, v, o, do, lse, scale, causal)
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    before = fa2.fa2_launch_count()
    rc = fa2.fa2_bwd_noalloc(q, k, v, o, do, lse, *got, scale, causal)
    assert rc == fa2.FA2_OK, fa2.status_string(rc)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    assert fa2.fa2_launch_count() - before == 3  # the kernels of one fa2_bwd call
    for g, r in zip(got, ref):
        assert torch.isfinite(g.float()).all()
        assert _close(g, r)
    # the same kernels: dK and dV are bitwise those of fa2_bwd
    assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])


# Each pair is two calls in a row on the shared buffer.  The second call has other
# inputs and a smaller problem than the first, so rows of the row statistics (D,
# LSE) or of the dQ accumulator left over by the first call would show up in the
# second call's results if the call did not rewrite everything it reads.
@pytest.mark.parametrize("first,second", [("workload_d64_causal", "b2h8_n500_d64"),
                                          ("b2h4_n700_d128_causal", "b1h3_n300_d128_causal")])
def test_noalloc_backward_matches_backward_twice(first, second):
    _noalloc_matches_backward(first)
    _noalloc_matches_backward(second)


def test_noalloc_backward_rejects_sizes_beyond_its_buffer():
    B, H, N, d = 1, 8, 16384, 64  # needs ~32.5 MiB of scratch (the dQ accumulator)
    assert fa2.fa2_bwd_workspace_size(B, H, N, d) > (32 << 20) - 256
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    k, v, o, do, dq, dk, dv = (torch.zeros_like(q) for _ in range(7))
    lse = torch.zeros(B, H, N, dtype=torch.float32, device="cuda")
    before = fa2.fa2_launch_count()
    rc = fa2.fa2_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, 0.1, False)
    assert rc == fa2.FA2_ERR_WORKSPACE
    assert fa2.fa2_launch_count() == before
