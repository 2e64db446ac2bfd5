"""GPU parity of the backward pass (fa2_bwd through the C ABI) against the fp64 oracle.

Tolerance (written here, from the problem statement): for each of dQ, dK, dV the
max-abs error is at most 1e-2 x max|reference|.  The GPU backward consumes the
GPU forward's O and LSE; the oracle recomputes everything from Q, K, V, dO in fp64.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

GRAD_REL = 1e-2
# Where the exact gradient is identically zero (N = 1: one key, so dS = P (dP - D)
# = 0) a bound of 1e-2 x max|ref| = 0 cannot be met by any rounded result: dP and
# D are two fp32 sums of the same d products taken in different orders.  The
# reference magnitude is floored at 1e-3, i.e. an absolute bound of 1e-5.
REF_FLOOR = 1e-3


def _gpu_fwd_bwd(x, scale, causal):
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, scale, causal)
    dq, dk, dv = fa2.backward(q, k, v, o, do, lse, scale, causal)
    rc, site = fa2.fa2_get_device_status()
    assert rc == fa2.FA2_OK, (fa2.status_string(rc), site)
    return dq.cpu(), dk.cpu(), dv.cpu()


def _check(got, ref, name, heads=None):
    g = got.double().numpy()
    if heads is not None:
        B, H = g.shape[:2]
        g = g.reshape(B * H, *g.shape[2:])[heads]
        ref = ref.reshape(B * H, *ref.shape[2:])[heads]
    scale = max(float(np.max(np.abs(ref))), REF_FLOOR)
    err = float(np.max(np.abs(g - ref)))
    assert np.isfinite(err) and err <= GRAD_REL * scale, f"{name}: err {err:.3e} vs max {scale:.3e}"


def _compare(x, scale, causal, heads=None):
    dq, dk, dv = _gpu_fwd_bwd(x, scale, causal)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], scale, causal, heads=heads)
    _check(dq, rq, "dQ", heads)
    _check(dk, rk, "dK", heads)
    _check(dv, rv, "dV", heads)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 255, 256, 300, 1000])
def test_bwd_small_shapes(N, d, causal, dtype):
    x = make_inputs(1, 2, N, d, dtype, seed=2000 + N + d, with_do=True)
    _compare(x, 1.0 / math.sqrt(d), causal)


def test_bwd_batch_heads_and_scale():
    x = make_inputs(2, 3, 384, 128, "bf16", seed=31, with_do=True)
    _compare(x, 0.2, True)
    _compare(x, 0.05, False)


def test_bwd_workload_fwdbwd_d64_causal_full():
    w = WORKLOADS["fwdbwd_bf16_b4h16_n1024_d64_causal"]
    _compare(workload_inputs(w), w.scale, w.causal)


def test_bwd_dk_dv_repeatable_and_dq_close():
    x = make_inputs(2, 2, 700, 128, "bf16", seed=32, with_do=True)
    runs = [_gpu_fwd_bwd(x, 0.1, True) for _ in range(3)]
    for dq, dk, dv in runs[1:]:
        assert torch.equal(dk, runs[0][1]) and torch.equal(dv, runs[0][2])
        # dQ sums fp32 partials with bulk reductions: order may change the last bits only
        assert torch.max(torch.abs(dq.float() - runs[0][0].float())) <= 1e-2 * torch.max(
            torch.abs(runs[0][0].float()))


def test_bwd_writes_nothing_outside_outputs():
    B, H, N, d = 1, 2, 200, 64
    x = make_inputs(B, H, N, d, "bf16", seed=33, with_do=True)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, 0.125, True)
    n, guard = B * H * N * d, 4096
    bufs = [torch.full((n + 2 * guard,), 5.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    dq, dk, dv = (b[guard:guard + n].view(B, H, N, d) for b in bufs)
    ws_bytes = fa2.fa2_bwd_workspace_size(B, H, N, d)
    wsbuf = torch.zeros(ws_bytes + 2 * guard, dtype=torch.uint8, device="cuda")
    ws = wsbuf[guard:guard + ws_bytes]
    assert fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, 0.125, True) == fa2.FA2_OK
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.all(b[:guard] == 5.0) and torch.all(b[guard + n:] == 5.0)
    assert torch.all(wsbuf[:guard] == 0) and torch.all(wsbuf[guard + ws_bytes:] == 0)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], 0.125, True)
    _check(dq.cpu(), rq, "dQ")
    _check(dk.cpu(), rk, "dK")
    _check(dv.cpu(), rv, "dV")


def test_bwd_rejects_small_workspace():
    x = make_inputs(1, 1, 128, 64, "bf16", seed=34, with_do=True)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, 0.125, False)
    ws = torch.empty(fa2.fa2_bwd_workspace_size(1, 1, 128, 64) - 256, dtype=torch.uint8,
                     device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    assert fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, 0.125, False) == fa2.FA2_ERR_WORKSPACE


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_repeated_runs_stay_correct(d, causal):
    """Timing-dependent races between the warp roles show up only in some runs: run
    the same backward several times and check every result."""
    x = make_inputs(1, 2, 1000, d, "bf16", seed=3000 + d + int(causal), with_do=True)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    scale = 1 / math.sqrt(d)
    o, lse = fa2.forward(q, k, v, scale, causal)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], scale, causal)
    for _ in range(8):
        dq, dk, dv = fa2.backward(q, k, v, o, do, lse, scale, causal)
        _check(dq.cpu(), rq, "dQ")
        _check(dk.cpu(), rk, "dK")
        _check(dv.cpu(), rv, "dV")
