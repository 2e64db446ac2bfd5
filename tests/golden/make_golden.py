"""Writes attn_small.json: tiny seeded attention problems with their fp64 results.

    python tests/golden/make_golden.py

The pages print no worked numeric example of the method, so nothing here comes
from them: the expected values are those of the fp64 oracle (the plain definition
of softmax attention, "Flash Attention spiegata: una guida completa", section
"Attention standard vs Flash attention": the fast method computes exactly
standard attention), written once by this script.  Only ``oracle`` computes them;
the inputs come from the seeded generator that every test uses.  The file lets
the CPU tests notice any change to the oracle's results and the GPU tests compare
the CUDA path with stored numbers without running the oracle.
"""

from __future__ import annotations

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from exact_io_aware_74_b200.workloads import make_inputs  # noqa: E402

CASES = [
    # name, B, H, N, d, causal, dtype, seed
    ("bf16_n5_d8_causal", 1, 2, 5, 8, True, "bf16", 4242),
    ("bf16_n5_d8", 1, 2, 5, 8, False, "bf16", 4243),
    ("fp16_n7_d16_causal", 1, 1, 7, 16, True, "fp16", 4244),
]


def build() -> dict:
    out = {"source": "fp64 oracle (oracle.attn_fwd_ref, oracle.attn_bwd_ref); inputs from "
                     "exact_io_aware_74_b200.workloads.make_inputs",
           "cases": []}
    for name, B, H, N, d, causal, dtype, seed in CASES:
        x = make_inputs(B, H, N, d, dtype, seed=seed, with_do=True)
        scale = 1.0 / d ** 0.5
        o, lse = oracle.attn_fwd_ref(x["q"], x["k"], x["v"], scale, causal)
        dq, dk, dv = oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], scale, causal)
        f = lambda t: t.double().numpy().tolist()  # 16-bit values, exact in fp64
        out["cases"].append({
            "name": name, "B": B, "H": H, "N": N, "d": d, "causal": causal, "dtype": dtype,
            "seed": seed, "scale": scale,
            "q": f(x["q"]), "k": f(x["k"]), "v": f(x["v"]), "do": f(x["do"]),
            "o": o.tolist(), "lse": lse.tolist(), "dq": dq.tolist(), "dk": dk.tolist(),
            "dv": dv.tolist(),
        })
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "attn_small.json"), "w") as fh:
        json.dump(build(), fh, indent=None, separators=(",", ":"))
        fh.write("\n")
    print("wrote", os.path.join(HERE, "attn_small.json"))
