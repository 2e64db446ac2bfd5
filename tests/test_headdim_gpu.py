"""GPU parity for head dims other than 64 and 128.

"Flash Attention spiegata: una guida completa", FlashAttention-2 section: the head
dimension goes up to 256.  Any multiple of 8 up to 256 runs in the forward (the
tiles are 64, 128, 192 or 256 columns wide and TMA reads zeros past d), and up to
128 in the backward.  Tolerances as for d = 64 / 128: O max-abs 2e-2 (bf16) /
5e-3 (fp16), LSE 1e-3, gradients 1e-2 x max|reference|.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_decode_inputs, make_inputs

pytestmark = pytest.mark.gpu

O_TOL = {"bf16": 2e-2, "fp16": 5e-3}
FWD_DIMS = [8, 32, 40, 72, 96, 112, 136, 160, 192, 200, 256]
BWD_DIMS = [8, 32, 40, 72, 96, 112]


def _fwd_check(x, scale, causal, dtype, window=None):
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    if window is None:
        o, lse = fa2.forward(q, k, v, scale, causal)
    else:
        o, lse = fa2.forward_window(q, k, v, scale, window)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    ro, rl = oracle.attn_fwd_ref(x["q"], x["k"], x["v"], scale, causal, window=window)
    assert np.max(np.abs(o.cpu().double().numpy() - ro)) <= O_TOL[dtype]
    assert np.max(np.abs(lse.cpu().double().numpy() - rl)) <= 1e-3


@pytest.mark.parametrize("d", FWD_DIMS)
@pytest.mark.parametrize("N,causal", [(1, True), (129, True), (300, False), (1000, True),
                                      (513, False)])
def test_fwd_head_dims_bf16(d, N, causal):
    x = make_inputs(1, 2, N, d, "bf16", seed=7000 + d + N)
    _fwd_check(x, 1 / math.sqrt(d), causal, "bf16")


@pytest.mark.parametrize("d", [32, 96, 160, 256])
def test_fwd_head_dims_fp16(d):
    x = make_inputs(2, 2, 700, d, "fp16", seed=7100 + d)
    _fwd_check(x, 1 / math.sqrt(d), True, "fp16")


@pytest.mark.parametrize("d", [96, 256])
def test_fwd_head_dims_window(d):
    x = make_inputs(1, 2, 1000, d, "bf16", seed=7200 + d)
    _fwd_check(x, 1 / math.sqrt(d), True, "bf16", window=300)


@pytest.mark.parametrize("d", [8, 96, 200, 256])
def test_fwd_head_dims_write_nothing_outside_outputs(d):
    B, H, N = 1, 3, 300
    x = make_inputs(B, H, N, d, "bf16", seed=7300 + d)
    n_o, n_l, guard = B * H * N * d, B * H * N, 4096
    obuf = torch.full((n_o + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((n_l + 2 * guard,), -3.0, dtype=torch.float32, device="cuda")
    o = obuf[guard:guard + n_o].view(B, H, N, d)
    lse = lbuf[guard:guard + n_l].view(B, H, N)
    q, k, v = (t.cuda() for t in (x["q"], x["k"], x["v"]))
    assert fa2.fa2_fwd(q, k, v, o, lse, d ** -0.5, True) == fa2.FA2_OK
    torch.cuda.synchronize()
    assert torch.all(obuf[:guard] == 7.0) and torch.all(obuf[guard + n_o:] == 7.0)
    assert torch.all(lbuf[:guard] == -3.0) and torch.all(lbuf[guard + n_l:] == -3.0)
    ro, _ = oracle.attn_fwd_ref(x["q"], x["k"], x["v"], d ** -0.5, True)
    assert np.max(np.abs(o.cpu().double().numpy() - ro)) <= O_TOL["bf16"]


def test_fwd_head_dims_repeatable():
    x = make_inputs(2, 3, 1000, 192, "bf16", seed=7400)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = fa2.forward(q, k, v, 0.07, True)
    o2, l2 = fa2.forward(q, k, v, 0.07, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [40, 96, 192, 256])
@pytest.mark.parametrize("Nq,Nk,sp", [(1, 3000, 4), (50, 2000, 3), (200, 1500, 2)])
def test_decode_head_dims(d, Nq, Nk, sp):
    x = make_decode_inputs(1, 3, Nq, Nk, d, "bf16", seed=7500 + d + Nq)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    for _ in range(3):
        o, lse = fa2.forward_decode(q, k, v, d ** -0.5, True, sp)
        assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
        ro, rl = oracle.attn_fwd_decode_ref(x["q"], x["k"], x["v"], d ** -0.5, True)
        assert np.max(np.abs(o.cpu().double().numpy() - ro)) <= O_TOL["bf16"]
        assert np.max(np.abs(lse.cpu().double().numpy() - rl)) <= 1e-3


def _grad_check(got, ref):
    scale = max(float(np.max(np.abs(ref))), 1e-3)
    assert float(np.max(np.abs(got.cpu().double().numpy() - ref))) <= 1e-2 * scale


@pytest.mark.parametrize("d", BWD_DIMS)
@pytest.mark.parametrize("N,causal", [(129, True), (300, False), (1000, True)])
def test_bwd_head_dims(d, N, causal):
    x = make_inputs(1, 2, N, d, "bf16", seed=7600 + d + N, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, s, causal)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, causal)
    for _ in range(2):
        dq, dk, dv = fa2.backward(q, k, v, o, do, lse, s, causal)
        assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
        _grad_check(dq, rq)
        _grad_check(dk, rk)
        _grad_check(dv, rv)


@pytest.mark.parametrize("d", [32, 96])
def test_bwd_head_dims_window_and_guard_bands(d):
    B, H, N = 1, 2, 700
    x = make_inputs(B, H, N, d, "bf16", seed=7700 + d, with_do=True)
    s = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward_window(q, k, v, s, 200)
    n, guard = B * H * N * d, 4096
    bufs = [torch.full((n + 2 * guard,), 5.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    dq, dk, dv = (b[guard:guard + n].view(B, H, N, d) for b in bufs)
    ws = torch.empty(fa2.fa2_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    rc = fa2.fa2_bwd_window(q, k, v, o, do, lse, dq, dk, dv, ws, s, 200)
    assert rc == fa2.FA2_OK and fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    for b in bufs:
        assert torch.all(b[:guard] == 5.0) and torch.all(b[guard + n:] == 5.0)
    rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], s, True, window=200)
    _grad_check(dq, rq)
    _grad_check(dk, rk)
    _grad_check(dv, rv)


def test_bwd_rejects_head_dims_above_128():
    x = make_inputs(1, 1, 64, 192, "bf16", seed=7800, with_do=True)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa2.forward(q, k, v, 0.1, False)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    assert fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, 0.1, False) == fa2.FA2_ERR_UNSUPPORTED


@pytest.mark.slow
@pytest.mark.parametrize("name", ["fwdbwd_bf16_b2h32_n8192_d96", "fwd_bf16_b2h16_n8192_d256"])
def test_headdim_workloads_full_size_sampled(name):
    """The measured head-dim workloads at full size: sampled forward rows of the
    last head against the oracle, and (d = 96) that head's whole backward."""
    from exact_io_aware_74_b200.workloads import WORKLOADS, workload_inputs
    w = WORKLOADS[name]
    x = workload_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa2.forward(q, k, v, w.scale, w.causal)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    bh = w.B * w.H - 1
    b, h = divmod(bh, w.H)
    rows = [0, 1, 127, 128, 4095, 4096, 8190, 8191]
    ro, rl = oracle.attn_fwd_rows_ref(x["q"], x["k"], x["v"], w.scale, w.causal, bh, rows)
    assert np.max(np.abs(o[b, h, rows].cpu().double().numpy() - ro)) <= O_TOL["bf16"]
    assert np.max(np.abs(lse[b, h, rows].cpu().double().numpy() - rl)) <= 1e-3
    if w.backward:
        do = x["do"].cuda()
        dq, dk, dv = fa2.backward(q, k, v, o, do, lse, w.scale, w.causal)
        assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
        rq, rk, rv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal,
                                         heads=[bh])
        for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
            _grad_check(got[b, h][None, None], ref[b, h][None, None])
