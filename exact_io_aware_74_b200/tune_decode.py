"""Times fa2_fwd_decode over split counts on one shape, to pick n_splits for a GPU.

    python -m exact_io_aware_74_b200.tune_decode B H Nq Nk d causal [splits ...]

Seeded N(0, 1) bf16 inputs.  Each split count is timed over back-to-back calls
(CUDA events around 30 queued calls after 3 warm-up calls), so host-side launch
work overlaps the device time as it does in a real decode loop.  Prints, per
split count, microseconds per call and the algorithmic HBM GB/s (Q, K, V read and
O, LSE written once), marking the library's own choice with '*'.
"""

from __future__ import annotations

import math
import sys

import torch

from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_decode_inputs

CALLS = 30


def time_splits(q, k, v, causal: bool, splits: int) -> float:
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    nws = fa2.fa2_fwd_decode_workspace_size(B, H, Nq, Nk, d, splits)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    scale = 1.0 / math.sqrt(d)

    def call():
        rc = fa2.fa2_fwd_decode(q, k, v, o, lse, scale, causal, splits, ws)
        if rc != fa2.FA2_OK:
            raise fa2.FA2Error(rc, "fa2_fwd_decode")

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(CALLS):
        call()
    b.record()
    b.synchronize()
    rc, site = fa2.fa2_get_device_status()
    if rc != fa2.FA2_OK:
        raise fa2.FA2Error(rc, f"device status (wait site {site})")
    return a.elapsed_time(b) * 1e3 / CALLS


def main(argv: list[str]) -> int:
    B, H, Nq, Nk, d, causal = (int(x) for x in argv[:6])
    auto = fa2.fa2_fwd_decode_splits(B, H, Nq, Nk, d)
    splits = [int(x) for x in argv[6:]] or sorted({1, 2, 4, 8, 16, 32, auto})
    x = make_decode_inputs(B, H, Nq, Nk, d, "bf16", seed=6)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    hbm = B * H * (2 * Nq * d * 2 + 2 * Nk * d * 2 + Nq * 4)
    for sp in splits:
        us = time_splits(q, k, v, bool(causal), sp)
        print(f"B={B} H={H} Nq={Nq} Nk={Nk} d={d} causal={causal} splits={sp:4d}"
              f"{'*' if sp == auto else ' '} {us:8.1f} us {hbm / us / 1e3:7.0f} GB/s", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
