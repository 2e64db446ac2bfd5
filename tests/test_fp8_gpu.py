"""GPU parity of the 8-bit forward (fa2_fwd_fp8) against the oracle.

"Flash Attention spiegata: una guida completa", FlashAttention-3 section: 8-bit
floating point for the matrix products.  Inputs are E4M3 codes with per-tensor
scales; the oracle is exact attention of their real values (oracle.attn_fwd_fp8_ref).

Tolerance, derived from the kernel's arithmetic.  Everything but P is fp32
(scores, row max, row sum, accumulation), so the error is dominated by rounding
P to E4M3 before P V.  With P taken relative to the row max (P_max = 1) the
rounding error of one probability is at most 2^-4 P in the normal range and at
most 2^-10 (half the subnormal spacing 2^-9) below 2^-6, scaled by P_max when the
kernel's running max lags the true one; the row sum uses the unrounded values.
So, per output element, with P normalised over the row:

    |O_gpu - O| <= sum_j max(2^-4 P_ij, 2^-10 max_j P_ij) |V_jc|  +  2^-8 |O_ic|  +  1e-3

(the middle term: rounding O to bf16; the last: fp32 accumulation and the scale
products).  LSE depends only on the fp32 path: 1e-3 as for 16-bit inputs.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_fp8_inputs

pytestmark = pytest.mark.gpu


def _codes(x):
    return {n: x[n].view(torch.uint8).numpy() for n in ("q", "k", "v")}


def _bound(codes, s, scale, causal):
    qd, kd, vd = (oracle.e4m3_decode(codes[n]) * s for n in ("q", "k", "v"))
    p = oracle.attn_probs_ref(qd, kd, scale, causal)
    pmax = p.max(axis=-1, keepdims=True)
    w = np.where(p > 0, np.maximum(2.0 ** -4 * p, 2.0 ** -10 * pmax), 0.0)
    return w @ np.abs(vd)


def _run_check(x, scale, causal):
    s = x["scale"]
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa2.forward_fp8(q, k, v, scale, causal, s, s, s)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    c = _codes(x)
    ro, rl = oracle.attn_fwd_fp8_ref(c["q"], c["k"], c["v"], scale, causal, s, s, s)
    err = np.abs(o.cpu().double().numpy() - ro)
    tol = _bound(c, s, scale, causal) + 2.0 ** -8 * np.abs(ro) + 1e-3
    assert np.all(err <= tol), float(np.max(err - tol))
    assert np.max(np.abs(lse.cpu().double().numpy() - rl)) <= 1e-3
    return o, err, tol


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [16, 64, 96, 128])
@pytest.mark.parametrize("N", [1, 100, 129, 300, 1000])
def test_fp8_forward(N, d, causal):
    x = make_fp8_inputs(1, 2, N, d, seed=9000 + N + d)
    _run_check(x, d ** -0.5, causal)


@pytest.mark.parametrize("scale", [0.02, 0.3, 1.0])
def test_fp8_forward_flat_and_peaked_rows(scale):
    """Flat rows (small scale) average many rounded probabilities; peaked rows
    (large scale) are dominated by one key, where a misplaced P column or V row
    would show at once."""
    x = make_fp8_inputs(2, 2, 700, 128, seed=9100)
    o, err, tol = _run_check(x, scale, True)
    # the typical error is far inside the worst-case bound
    assert float(np.median(err / tol)) < 0.25


def test_fp8_matches_16bit_path_on_the_same_values():
    """E4M3 values are exact in bf16: the 16-bit path on the decoded inputs differs
    from the 8-bit path only by P's rounding (E4M3 against bf16)."""
    x = make_fp8_inputs(1, 4, 1000, 128, seed=9200)
    s = x["scale"]
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o8, l8 = fa2.forward_fp8(q, k, v, 0.09, True, s, s, s)
    qb, kb, vb = ((t.to(torch.float32) * s).to(torch.bfloat16) for t in (q, k, v))
    o16, l16 = fa2.forward(qb, kb, vb, 0.09, True)
    assert torch.max(torch.abs(l8 - l16)).item() <= 1e-3
    c = _codes(x)
    tol = _bound(c, s, 0.09, True) + 2.0 ** -7 * np.abs(o16.cpu().double().numpy()) + 2e-3
    assert np.all(np.abs((o8.float() - o16.float()).cpu().double().numpy()) <= tol)


def test_fp8_repeatable_and_guard_bands():
    B, H, N, d = 1, 3, 500, 64
    x = make_fp8_inputs(B, H, N, d, seed=9300)
    s = x["scale"]
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    n_o, n_l, guard = B * H * N * d, B * H * N, 4096
    obuf = torch.full((n_o + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((n_l + 2 * guard,), -3.0, dtype=torch.float32, device="cuda")
    o = obuf[guard:guard + n_o].view(B, H, N, d)
    lse = lbuf[guard:guard + n_l].view(B, H, N)
    assert fa2.fa2_fwd_fp8(q, k, v, o, lse, 0.125, True, s, s, s) == fa2.FA2_OK
    torch.cuda.synchronize()
    assert torch.all(obuf[:guard] == 7.0) and torch.all(obuf[guard + n_o:] == 7.0)
    assert torch.all(lbuf[:guard] == -3.0) and torch.all(lbuf[guard + n_l:] == -3.0)
    o2, l2 = fa2.forward_fp8(q, k, v, 0.125, True, s, s, s)
    assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_fp8_scales_apply():
    """Doubling v_scale doubles O; q_scale * k_scale and scale are interchangeable."""
    x = make_fp8_inputs(1, 2, 300, 128, seed=9400)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    s = x["scale"]
    o1, l1 = fa2.forward_fp8(q, k, v, 0.1, False, s, s, s)
    o2, l2 = fa2.forward_fp8(q, k, v, 0.1, False, s, s, 2 * s)
    assert torch.equal(o2.float(), 2 * o1.float()) and torch.equal(l1, l2)
    o3, l3 = fa2.forward_fp8(q, k, v, 0.2, False, s / 2, s, s)
    assert torch.max(torch.abs(o3.float() - o1.float())).item() <= 1e-2
    assert torch.max(torch.abs(l3 - l1)).item() <= 1e-5


@pytest.mark.slow
def test_fp8_workload_full_size_sampled():
    from exact_io_aware_74_b200.workloads import FP8_WORKLOADS
    w = FP8_WORKLOADS["fwd_e4m3_b2h32_n8192_d128"]
    x = make_fp8_inputs(w.B, w.H, w.N, w.d, seed=w.seed)
    s = x["scale"]
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa2.forward_fp8(q, k, v, w.scale, w.causal, s, s, s)
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    bh = w.B * w.H - 1
    b, h = divmod(bh, w.H)
    rows = [0, 1, 127, 128, 4095, 8191]
    c = _codes(x)
    qd, kd, vd = (oracle.e4m3_decode(c[n]) * s for n in ("q", "k", "v"))
    ro, rl = oracle.attn_fwd_rows_ref(qd, kd, vd, w.scale, w.causal, bh, rows)
    # per-row bound from that head's exact probabilities
    sc = w.scale * qd[b, h, rows] @ kd[b, h].T
    p = np.exp(sc - sc.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    wgt = np.maximum(2.0 ** -4 * p, 2.0 ** -10 * p.max(axis=1, keepdims=True))
    tol = wgt @ np.abs(vd[b, h]) + 2.0 ** -8 * np.abs(ro) + 1e-3
    assert np.all(np.abs(o[b, h, rows].cpu().double().numpy() - ro) <= tol)
    assert np.max(np.abs(lse[b, h, rows].cpu().double().numpy() - rl)) <= 1e-3
