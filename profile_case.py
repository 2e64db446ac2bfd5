"""Runs fa2_fwd (and fa2_bwd), or fa2_fwd_decode, a few times on one shape, for profilers.

    python profile_case.py B H N d causal [reps] [--fwd-only]
    python profile_case.py --decode B H Nq Nk d causal [reps] [splits]
    python profile_case.py --fp8 B H N d causal [reps]

Seeded N(0, 1) bf16 inputs; exits non-zero if a call or the device status fails.
Used to capture Nsight Compute profiles of one kernel on a small case.  With
--decode, splits = 0 (the default) takes the library's split count.
"""

from __future__ import annotations

import math
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import torch

from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_decode_inputs, make_fp8_inputs, make_inputs


def decode(args: list[str]) -> int:
    B, H, Nq, Nk, d, causal = (int(a) for a in args[:6])
    reps = int(args[6]) if len(args) > 6 else 2
    splits = int(args[7]) if len(args) > 7 else 0
    x = make_decode_inputs(B, H, Nq, Nk, d, "bf16", seed=5)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    for _ in range(reps):
        fa2.forward_decode(q, k, v, 1.0 / math.sqrt(d), bool(causal), splits)
    rc, site = fa2.fa2_get_device_status()
    print(f"status {fa2.status_string(rc)} site {site}")
    return 0 if rc == fa2.FA2_OK else 1


def fp8(args: list[str]) -> int:
    B, H, N, d, causal = (int(a) for a in args[:5])
    reps = int(args[5]) if len(args) > 5 else 2
    x = make_fp8_inputs(B, H, N, d, seed=5)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    s = x["scale"]
    for _ in range(reps):
        fa2.forward_fp8(q, k, v, 1.0 / math.sqrt(d), bool(causal), s, s, s)
    rc, site = fa2.fa2_get_device_status()
    print(f"status {fa2.status_string(rc)} site {site}")
    return 0 if rc == fa2.FA2_OK else 1


def main(argv: list[str]) -> int:
    if "--decode" in argv:
        return decode([a for a in argv if not a.startswith("--")])
    if "--fp8" in argv:
        return fp8([a for a in argv if not a.startswith("--")])
    fwd_only = "--fwd-only" in argv
    args = [a for a in argv if not a.startswith("--")]
    B, H, N, d, causal = (int(a) for a in args[:5])
    reps = int(args[5]) if len(args) > 5 else 2
    x = make_inputs(B, H, N, d, "bf16", seed=5, with_do=not fwd_only)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    do = None if fwd_only else x["do"].cuda()
    scale = 1.0 / math.sqrt(d)
    for _ in range(reps):
        o, lse = fa2.forward(q, k, v, scale, bool(causal))
        if not fwd_only:
            fa2.backward(q, k, v, o, do, lse, scale, bool(causal))
    rc, site = fa2.fa2_get_device_status()
    print(f"status {fa2.status_string(rc)} site {site}")
    return 0 if rc == fa2.FA2_OK else 1


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
