"""GPU parity of the backward's persistent tile scheduler.

The backward runs at most one CTA per SM; each CTA starts with one key tile and
then takes the next free one from a counter in the workspace, carrying its barrier
phases, its (Q, dO) ring, its K/V buffers and its tile ring from one tile to the
next.  Small problems have fewer tiles than SMs, so the test hook
``fa2_debug_set_bwd_grid`` caps the grid to make every CTA run many tiles: one CTA
running all of them, and counts that do not divide the tile count.  dK and dV of a key tile do not depend on which
CTA computed them (bitwise equal to the uncapped run); dQ is summed by float
reductions whose order may change (checked against the oracle).  Tolerances as
elsewhere: gradients 1e-2 x max|reference|.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


def _grad_check(got, ref):
    scale = max(float(np.max(np.abs(ref))), 1e-3)
    assert float(np.max(np.abs(got.cpu().double().numpy() - ref))) <= 1e-2 * scale


def _run(q, k, v, o, do, lse, s, causal, window, max_ctas):
    fa2.fa2_debug_set_bwd_grid(max_ctas)
    try:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(fa2.fa2_bwd_workspace_size(*q.shape), dtype=torch.uint8, device="cuda")
        if window is None:
            rc = fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, s, causal)
        else:
            rc = fa2.fa2_bwd_window(q, k, v, o, do, lse, dq, dk, dv, ws, s, window)
        assert rc == fa2.FA2_OK
        assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
        return dq, dk, dv
    finally:
        fa2.fa2_debug_set_bwd_grid(0)


@pytest.mark.parametrize("d", [64, 128, 96])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("max_ctas", [1, 2, 5, 7])
def test_bwd_capped_grid_matches_oracle_and_uncapped(d, causal, max_ctas):
    B, H, N = 1, 3, 700  # 6 key tiles per head (the last ragged): 18 tiles
    x = make_inputs(B, H, N, d, "bf16", seed=9900 + d + max_ctas + 50 * causal, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, s, causal)
    ref = _run(q, k, v, o, do, lse, s, causal, None, 0)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, causal)
    for _ in range(2):
        dq, dk, dv = _run(q, k, v, o, do, lse, s, causal, None, max_ctas)
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
        _grad_check(dq, rq)
        _grad_check(dk, rk)
        _grad_check(dv, rv)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("max_ctas", [1, 3])
def test_bwd_capped_grid_sliding_window(d, max_ctas):
    B, H, N, W = 2, 2, 1000, 200
    x = make_inputs(B, H, N, d, "bf16", seed=9950 + d + max_ctas, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward_window(q, k, v, s, W)
    dq, dk, dv = _run(q, k, v, o, do, lse, s, True, W, max_ctas)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, True, window=W)
    _grad_check(dq, rq)
    _grad_check(dk, rk)
    _grad_check(dv, rv)


def test_bwd_capped_grid_fp16_many_tiles_per_cta():
    # 2 x 4 heads x 9 key tiles = 72 tiles on 4 CTAs: 18 tiles each
    B, H, N, d = 2, 4, 1100, 64
    x = make_inputs(B, H, N, d, "fp16", seed=9970, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, s, True)
    dq, dk, dv = _run(q, k, v, o, do, lse, s, True, None, 4)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, True)
    _grad_check(dq, rq)
    _grad_check(dk, rk)
    _grad_check(dv, rv)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_capped_grid_timeout_reports_and_recovers(d):
    B, H, N = 1, 2, 900
    x = make_inputs(B, H, N, d, "bf16", seed=9980 + d, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, s, True)
    fa2.fa2_debug_set(1, 50)
    try:
        fa2.fa2_debug_set_bwd_grid(2)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(fa2.fa2_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
        assert fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, s, True) == fa2.FA2_OK
        status, site = fa2.fa2_get_device_status()
    finally:
        fa2.fa2_debug_set(0, 0)
        fa2.fa2_debug_set_bwd_grid(0)
    assert status == fa2.FA2_ERR_TIMEOUT and site >= 32
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    dq, dk, dv = _run(q, k, v, o, do, lse, s, True, None, 2)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, True)
    _grad_check(dq, rq)
    _grad_check(dk, rk)
    _grad_check(dv, rv)
