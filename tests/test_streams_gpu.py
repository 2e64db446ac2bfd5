"""The calls on user streams and inside CUDA graphs.

Every entry point enqueues on the stream it is given and returns; the backward's
three kernels and the decode merge are chained by programmatic dependent launch.
These tests check that the results are ordered correctly against other work on
the same stream, that two streams can run calls at once, and that a captured
graph of forward + backward + decode replays to the eager results.
"""

import math

import pytest
import torch

from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_decode_inputs, make_inputs

pytestmark = pytest.mark.gpu


def _problem(seed, B=2, H=4, N=700, d=64):
    x = make_inputs(B, H, N, d, "bf16", seed=seed, with_do=True)
    return [x[n].cuda() for n in ("q", "k", "v", "do")]


def _fwd_bwd(q, k, v, do, stream, ws=None):
    d = q.shape[-1]
    s = 1 / math.sqrt(d)
    o, lse = torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if ws is None:
        ws = torch.empty(fa2.fa2_bwd_workspace_size(*q.shape), dtype=torch.uint8, device="cuda")
    assert fa2.fa2_fwd(q, k, v, o, lse, s, True, stream) == fa2.FA2_OK
    assert fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, s, True, stream) == fa2.FA2_OK
    return o, lse, dq, dk, dv


def test_calls_on_a_side_stream_are_ordered_with_other_work():
    q, k, v, do = _problem(9800)
    ref = _fwd_bwd(q, k, v, do, None)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    q2 = torch.empty_like(q)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # the input is produced by other work on the same stream just before the call,
        # and the outputs are consumed by other work just after
        q2.copy_(q * 2)
        q2.mul_(0.5)
        got = _fwd_bwd(q2, k, v, do, s)
        sums = [t.float().sum() for t in got]
    s.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b) or a.dtype == torch.bfloat16 and \
            torch.max(torch.abs(a.float() - b.float())).item() <= 1e-2 * max(b.float().abs().max().item(), 1e-3)
    assert all(torch.isfinite(x) for x in sums)
    assert fa2.fa2_get_device_status(s) == (fa2.FA2_OK, 0)


def test_two_streams_run_independent_problems():
    p1, p2 = _problem(9801), _problem(9802, N=1000, d=128)
    r1, r2 = _fwd_bwd(*p1, None), _fwd_bwd(*p2, None)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            a = _fwd_bwd(*p1, s1)
        with torch.cuda.stream(s2):
            b = _fwd_bwd(*p2, s2)
        outs.append((a, b))
    torch.cuda.synchronize()
    for a, b in outs:
        # forward bitwise repeatable; dK, dV too; dQ (float atomics) to the last bits
        for got, ref in ((a, r1), (b, r2)):
            assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
            assert torch.equal(got[3], ref[3]) and torch.equal(got[4], ref[4])
            assert torch.max(torch.abs(got[2].float() - ref[2].float())).item() <= \
                1e-2 * ref[2].float().abs().max().item()
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)


def test_cuda_graph_capture_replays_forward_backward_and_decode():
    q, k, v, do = _problem(9803)
    xd = make_decode_inputs(1, 8, 1, 4096, 128, "bf16", seed=9804)
    qd, kd, vd = (xd[n].cuda() for n in ("q", "k", "v"))
    sp = 4
    wsd = torch.empty(fa2.fa2_fwd_decode_workspace_size(1, 8, 1, 4096, 128, sp), dtype=torch.uint8,
                      device="cuda")
    od = torch.empty_like(qd)
    lsed = torch.empty((1, 8, 1), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa2.fa2_bwd_workspace_size(*q.shape), dtype=torch.uint8, device="cuda")

    # eager references (these first calls also do the library's one-time set-up)
    ref = [t.clone() for t in _fwd_bwd(q, k, v, do, None, ws)]
    assert fa2.fa2_fwd_decode(qd, kd, vd, od, lsed, 0.1, True, sp, wsd) == fa2.FA2_OK
    ref_d = (od.clone(), lsed.clone())
    torch.cuda.synchronize()

    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        outs = _fwd_bwd(q, k, v, do, s, ws)
        assert fa2.fa2_fwd_decode(qd, kd, vd, od, lsed, 0.1, True, sp, wsd, s) == fa2.FA2_OK
    for _ in range(3):
        for t in list(outs) + [od, lsed]:
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(outs[0], ref[0]) and torch.equal(outs[1], ref[1])
        assert torch.equal(outs[3], ref[3]) and torch.equal(outs[4], ref[4])
        assert torch.max(torch.abs(outs[2].float() - ref[2].float())).item() <= \
            1e-2 * ref[2].float().abs().max().item()
        assert torch.equal(od, ref_d[0]) and torch.equal(lsed, ref_d[1])
    assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)
    del g
