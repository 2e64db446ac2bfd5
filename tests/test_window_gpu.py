"""GPU parity of the sliding-window calls (fa2_fwd_window / fa2_bwd_window).

Reading of "Flash Attention 2: attivarla (llama.cpp, Ollama, vLLM)", section
"Modelli con attenzione a finestra scorrevole non standard": query i sees its
``window`` most recent keys, max(0, i - window + 1) .. i.  Tolerances as for the
plain calls: O max-abs 2e-2 (bf16) / 5e-3 (fp16), LSE 1e-3, gradients
1e-2 x max|reference| (floored at 1e-3 for exactly-zero references).
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

O_TOL = {"bf16": 2e-2, "fp16": 5e-3}


def _fwd(x, scale, window):
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa2.forward_window(q, k, v, scale, window)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,W", [(1, 1), (100, 7), (300, 1), (300, 64), (300, 128), (300, 129),
                                 (1000, 200), (1000, 513), (700, 700), (777, 2000)])
def test_fwd_window(N, W, d, dtype):
    x = make_inputs(1, 2, N, d, dtype, seed=4000 + N + W + d)
    s = 1 / math.sqrt(d)
    o, lse = _fwd(x, s, W)
    ro, rl = oracle.attn_fwd_ref(x["q"], x["k"], x["v"], s, True, window=W)
    assert np.max(np.abs(o.double().numpy() - ro)) <= O_TOL[dtype]
    assert np.max(np.abs(lse.double().numpy() - rl)) <= 1e-3


def test_fwd_window_at_least_n_equals_causal():
    x = make_inputs(2, 2, 513, 128, "bf16", seed=41)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = fa2.forward_window(q, k, v, 0.1, 513)
    o2, l2 = fa2.forward(q, k, v, 0.1, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_window_one_is_identity():
    x = make_inputs(1, 3, 400, 64, "fp16", seed=42)
    o, lse = _fwd(x, 0.125, 1)
    assert torch.max(torch.abs(o.float() - x["v"].float())) <= O_TOL["fp16"]


def _check_grad(got, ref):
    scale = max(float(np.max(np.abs(ref))), 1e-3)
    assert float(np.max(np.abs(got.double().numpy() - ref))) <= 1e-2 * scale


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,W", [(100, 7), (300, 64), (300, 129), (1000, 200), (1000, 513),
                                 (777, 2000)])
def test_bwd_window(N, W, d):
    x = make_inputs(1, 2, N, d, "bf16", seed=5000 + N + W + d, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward_window(q, k, v, s, W)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, True, window=W)
    for _ in range(3):  # repeated: races between the warp roles show up only in some runs
        dq, dk, dv = fa2.backward_window(q, k, v, o, do, lse, s, W)
        assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
        _check_grad(dq.cpu(), rq)
        _check_grad(dk.cpu(), rk)
        _check_grad(dv.cpu(), rv)


def test_window_rejects_bad_window():
    x = make_inputs(1, 1, 64, 64, "bf16", seed=43, with_do=True)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 64), dtype=torch.float32, device="cuda")
    assert fa2.fa2_fwd_window(q, k, v, o, lse, 0.1, 0) == fa2.FA2_ERR_INVALID_ARG
    ws = torch.empty(fa2.fa2_bwd_workspace_size(1, 1, 64, 64), dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    assert fa2.fa2_bwd_window(q, k, v, o, do, lse, dq, dk, dv, ws, 0.1, -3) == fa2.FA2_ERR_INVALID_ARG


@pytest.mark.slow
def test_window_workload_full_size_sampled():
    """The measured sliding-window workload at full size: sampled forward rows and
    one whole head of the backward against the oracle."""
    from exact_io_aware_74_b200.workloads import WORKLOADS, workload_inputs
    w = WORKLOADS["fwdbwd_bf16_b8h16_n4096_d128_window1024"]
    x = workload_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward_window(q, k, v, w.scale, w.window)
    dq, dk, dv = fa2.backward_window(q, k, v, o, do, lse, w.scale, w.window)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    rows = [0, 1, 1023, 1024, 1025, 2047, 3000, 4095]
    bh = w.B * w.H - 1
    ro, rl = oracle.attn_fwd_rows_ref(x["q"], x["k"], x["v"], w.scale, True, bh, rows,
                                      window=w.window)
    b, h = divmod(bh, w.H)
    assert np.max(np.abs(o[b, h, rows].cpu().double().numpy() - ro)) <= O_TOL["bf16"]
    assert np.max(np.abs(lse[b, h, rows].cpu().double().numpy() - rl)) <= 1e-3
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], w.scale, True,
                                     heads=[bh], window=w.window)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        _check_grad(got[b, h].cpu()[None, None], ref[b, h][None, None])
