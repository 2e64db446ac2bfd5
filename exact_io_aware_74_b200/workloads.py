"""Seeded synthetic attention inputs and the named workloads.

This module holds no attention arithmetic: it draws Gaussian tensors from a
seeded CPU generator and applies the power-of-two scalings the workloads ask
for.  The same host tensors feed the CUDA path (after one copy to the device)
and the CPU oracle (after an exact upcast to fp64), so both sides see identical
16-bit values.

Recipe (the same for every workload):
  * ``torch.Generator('cpu').manual_seed(seed)``;
  * ``randn`` in fp32, shape [B, H, N, d], drawn in the order Q, K, V, dO;
  * optional multiplication of every input by ``input_scale`` (a power of two,
    so exact before rounding);
  * optional key outliers: per (batch, head), ceil(frac * N) distinct key rows
    chosen with ``randperm`` from the same generator, drawn after dO, are
    multiplied by ``outlier_mult`` (a power of two);
  * a cast to the 16-bit dtype with round-to-nearest-even.

The attention pages measure on model training and local LLM inference, which
need trained weights; these Gaussian tensors of the same shapes (sequence
lengths 128 .. 32768, head dims 64 and 128) stand in for them.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str
    causal: bool
    seed: int
    backward: bool = False
    input_scale: float = 1.0
    outlier_frac: float = 0.0
    outlier_mult: float = 8.0
    window: int = 0  # sliding window (causal only): row i sees its `window` most recent keys
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: two N x N x d products, halved when causal.

        With a sliding window W the products cover the sum over rows of the keys
        each row sees, min(i + 1, W), instead of N^2 / 2.
        """
        if self.window:
            w, n = min(self.window, self.N), self.N
            pairs = w * (w + 1) / 2.0 + (n - w) * w
            return 4.0 * self.B * self.H * self.d * pairs
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    @property
    def bwd_flops(self) -> float:
        """Algorithmic backward FLOPs: five products, i.e. 2.5 x forward."""
        return 2.5 * self.fwd_flops


WORKLOADS = {
    "fwd_fp16_b1h2_n128_d64": Workload(
        "fwd_fp16_b1h2_n128_d64", 1, 2, 128, 64, "fp16", False, 0,
        note="small forward, fp16, non-causal"),
    "fwdbwd_bf16_b4h16_n1024_d64_causal": Workload(
        "fwdbwd_bf16_b4h16_n1024_d64_causal", 4, 16, 1024, 64, "bf16", True, 1, backward=True,
        note="forward + backward, causal, head dim 64"),
    "fwd_bf16_b2h32_n8192_d128": Workload(
        "fwd_bf16_b2h32_n8192_d128", 2, 32, 8192, 128, "bf16", False, 2,
        note="compute-bound forward, non-causal"),
    "fwdbwd_bf16_b8h16_n4096_d128_causal": Workload(
        "fwdbwd_bf16_b8h16_n4096_d128_causal", 8, 16, 4096, 128, "bf16", True, 3, backward=True,
        input_scale=0.5, note="training shape, causal, inputs x0.5"),
    "fwd_bf16_b1h32_n32768_d128_causal_outliers": Workload(
        "fwd_bf16_b1h32_n32768_d128_causal_outliers", 1, 32, 32768, 128, "bf16", True, 4,
        outlier_frac=0.01, outlier_mult=8.0,
        note="long-context causal forward, 1% of key rows x8 per head"),
    # Not one of the five headline workloads: the sliding-window row, measured on
    # the training shape with a 1024-key window.
    "fwdbwd_bf16_b8h16_n4096_d128_window1024": Workload(
        "fwdbwd_bf16_b8h16_n4096_d128_window1024", 8, 16, 4096, 128, "bf16", True, 5,
        backward=True, input_scale=0.5, window=1024,
        note="training shape with a sliding window of 1024 keys"),
    # Head dims other than 64 / 128: the headline shape at d = 96 (forward and
    # backward, 128-wide tiles) and the forward at d = 256 (one query tile per CTA).
    "fwdbwd_bf16_b2h32_n8192_d96": Workload(
        "fwdbwd_bf16_b2h32_n8192_d96", 2, 32, 8192, 96, "bf16", False, 7, backward=True,
        note="headline shape at head dim 96"),
    "fwd_bf16_b2h16_n8192_d256": Workload(
        "fwd_bf16_b2h16_n8192_d256", 2, 16, 8192, 256, "bf16", False, 8,
        note="forward at head dim 256"),
}

# 8-bit forward (E4M3 Q, K, V; bf16 O) on the headline shape.  Inputs from
# make_fp8_inputs; FLOPs counted as for the 16-bit forward.
FP8_WORKLOADS = {
    "fwd_e4m3_b2h32_n8192_d128": Workload(
        "fwd_e4m3_b2h32_n8192_d128", 2, 32, 8192, 128, "e4m3", False, 9,
        note="headline shape with E4M3 inputs"),
}

WORKLOAD_ORDER = list(WORKLOADS)


def make_inputs(B: int, H: int, N: int, d: int, dtype: str, seed: int, *,
                with_do: bool = False, input_scale: float = 1.0,
                outlier_frac: float = 0.0, outlier_mult: float = 8.0) -> dict:
    """Seeded host tensors q, k, v (and do) of shape [B,H,N,d] in ``dtype``.

    Also returns ``outlier_rows`` ([B,H,n_out] int64 key-row indices, possibly
    empty) so tests can check the outliers are where the recipe puts them.
    """
    if dtype not in DTYPES:
        raise ValueError(f"dtype must be one of {sorted(DTYPES)}")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32) if with_do else None
    if input_scale != 1.0:
        q.mul_(input_scale)
        k.mul_(input_scale)
        v.mul_(input_scale)
        if do is not None:
            do.mul_(input_scale)
    n_out = int(math.ceil(outlier_frac * N)) if outlier_frac > 0 else 0
    rows = torch.empty((B, H, n_out), dtype=torch.int64)
    if n_out:
        for b in range(B):
            for h in range(H):
                idx = torch.randperm(N, generator=g)[:n_out]
                rows[b, h] = idx
                k[b, h, idx] *= outlier_mult
    t = DTYPES[dtype]
    out = {"q": q.to(t), "k": k.to(t), "v": v.to(t), "outlier_rows": rows}
    if do is not None:
        out["do"] = do.to(t)
    return out


@dataclass(frozen=True)
class DecodeWorkload:
    """Nq query rows (the last Nq positions) against Nk key/value rows."""
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    dtype: str
    causal: bool
    seed: int
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def pairs(self) -> int:
        """(query, key) pairs one head scores: query i sees Nk - Nq + i + 1 keys when
        causal (bottom-right alignment), all Nk otherwise."""
        if not self.causal:
            return self.Nq * self.Nk
        return self.Nq * (self.Nk - self.Nq) + self.Nq * (self.Nq + 1) // 2

    @property
    def fwd_flops(self) -> float:
        return 4.0 * self.B * self.H * self.d * self.pairs

    @property
    def hbm_bytes(self) -> int:
        """Algorithmic HBM bytes of one call: Q, K, V read once, O and LSE written once."""
        e = 2  # 16-bit elements
        bh = self.B * self.H
        return bh * (self.Nq * self.d * e * 2 + self.Nk * self.d * e * 2 + self.Nq * 4)


DECODE_WORKLOADS = {
    # One decode step after the long-context prompt: one new query per head
    # against a 32768-entry key/value cache (512 MiB of K and V, beyond L2).
    "decode_bf16_b1h32_nq1_nk32768_d128": DecodeWorkload(
        "decode_bf16_b1h32_nq1_nk32768_d128", 1, 32, 1, 32768, 128, "bf16", True, 6,
        note="decode step: 1 query per head against a 32768-key cache"),
}


def make_decode_inputs(B: int, H: int, Nq: int, Nk: int, d: int, dtype: str, seed: int) -> dict:
    """Seeded host tensors q [B,H,Nq,d] and k, v [B,H,Nk,d] in ``dtype``: the same
    recipe as ``make_inputs`` (N(0,1), drawn in the order Q, K, V)."""
    if dtype not in DTYPES:
        raise ValueError(f"dtype must be one of {sorted(DTYPES)}")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    t = DTYPES[dtype]
    return {"q": q.to(t), "k": k.to(t), "v": v.to(t)}


def decode_inputs(w: DecodeWorkload) -> dict:
    return make_decode_inputs(w.B, w.H, w.Nq, w.Nk, w.d, w.dtype, w.seed)


def make_fp8_inputs(B: int, H: int, N: int, d: int, seed: int, amp: float = 16.0) -> dict:
    """Seeded E4M3 inputs: N(0, 1) draws (Q, K, V in that order) times ``amp`` (a
    power of two, so that small values keep their precision and |x| stays far
    below 448), cast to torch.float8_e4m3fn (round to nearest even).  The real
    values are the codes times ``scale`` = 1 / amp, returned for each tensor."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    out = {}
    for name in ("q", "k", "v"):
        x = torch.randn(shape, generator=g, dtype=torch.float32) * amp
        out[name] = x.to(torch.float8_e4m3fn)
    out["scale"] = 1.0 / amp
    return out


def workload_inputs(w: Workload, *, with_do: bool | None = None, B: int | None = None,
                    H: int | None = None) -> dict:
    """Inputs of a named workload (optionally with fewer batches / heads)."""
    return make_inputs(B or w.B, H or w.H, w.N, w.d, w.dtype, w.seed,
                       with_do=w.backward if with_do is None else with_do,
                       input_scale=w.input_scale, outlier_frac=w.outlier_frac,
                       outlier_mult=w.outlier_mult)
