"""Failure detection without a GPU fault: the test hook (fa2_debug_set) skips a
tile load, so a consumer's bounded wait runs out.  The kernels must report
FA2_ERR_TIMEOUT with a wait-site id through fa2_get_device_status, leave every
role through bounded waits (nothing traps, nothing hangs), and leave the context
usable: the next call computes correctly.  (The plain forward's case is in
test_fwd_gpu.py.)
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_decode_inputs, make_fp8_inputs, make_inputs

pytestmark = pytest.mark.gpu

WAIT_MS = 50


def _with_fault(call):
    fa2.fa2_debug_set(1, WAIT_MS)
    try:
        rc = call()
        status, site = fa2.fa2_get_device_status()
    finally:
        fa2.fa2_debug_set(0, 0)
    return rc, status, site


def _grad_check(got, ref):
    scale = max(float(np.max(np.abs(ref))), 1e-3)
    assert float(np.max(np.abs(got.cpu().double().numpy() - ref))) <= 1e-2 * scale


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", ["default", "noalloc", "deterministic"])
def test_bwd_timeout_path_reports_and_recovers(d, mode):
    B, H, N = 1, 2, 300
    x = make_inputs(B, H, N, d, "bf16", seed=9500 + d, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, s, True)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa2.fa2_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")

    def call():
        if mode == "noalloc":
            return fa2.fa2_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, s, True)
        if mode == "deterministic":
            return fa2.fa2_bwd_ex(q, k, v, o, do, lse, dq, dk, dv, ws, s, True, 0,
                                  fa2.FA2_BWD_DETERMINISTIC)
        return fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, s, True)

    rc, status, site = _with_fault(call)
    assert rc == fa2.FA2_OK
    assert status == fa2.FA2_ERR_TIMEOUT and site >= 32  # a backward wait site
    # the status word was cleared and the context still works
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    assert call() == fa2.FA2_OK
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, True)
    _grad_check(dq, rq)
    _grad_check(dk, rk)
    _grad_check(dv, rv)


def test_decode_timeout_path_reports_and_recovers():
    x = make_decode_inputs(1, 2, 1, 2000, 128, "bf16", seed=9600)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 1), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa2.fa2_fwd_decode_workspace_size(1, 2, 1, 2000, 128, 3), dtype=torch.uint8,
                     device="cuda")
    call = lambda: fa2.fa2_fwd_decode(q, k, v, o, lse, 0.1, True, 3, ws)
    rc, status, site = _with_fault(call)
    assert rc == fa2.FA2_OK and status == fa2.FA2_ERR_TIMEOUT and 0 < site < 32
    assert call() == fa2.FA2_OK
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    ro, rl = oracle.attn_fwd_decode_ref(x["q"], x["k"], x["v"], 0.1, True)
    assert np.max(np.abs(o.cpu().double().numpy() - ro)) <= 2e-2
    assert np.max(np.abs(lse.cpu().double().numpy() - rl)) <= 1e-3


def test_fp8_timeout_path_reports_and_recovers():
    x = make_fp8_inputs(1, 2, 500, 128, seed=9700)
    s = x["scale"]
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o = torch.empty((1, 2, 500, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 2, 500), dtype=torch.float32, device="cuda")
    call = lambda: fa2.fa2_fwd_fp8(q, k, v, o, lse, 0.09, False, s, s, s)
    rc, status, site = _with_fault(call)
    assert rc == fa2.FA2_OK and status == fa2.FA2_ERR_TIMEOUT and 0 < site < 32
    assert call() == fa2.FA2_OK
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    codes = {n: x[n].view(torch.uint8).numpy() for n in ("q", "k", "v")}
    _, rl = oracle.attn_fwd_fp8_ref(codes["q"], codes["k"], codes["v"], 0.09, False, s, s, s)
    assert np.max(np.abs(lse.cpu().double().numpy() - rl)) <= 1e-3
