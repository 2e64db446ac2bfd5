"""Per-(batch, head) comparison of full-size GPU results with the fp64 oracle, spread
over a pool of host processes.

The pool is created with the ``spawn`` start method (a process forked after the
CUDA context exists can hang), and every worker limits its BLAS threads so that
the workers together use the host's cores once.  Workers receive one slice's
inputs and the GPU's results for it as float32 NumPy arrays (exact for 16-bit
values), run the oracle on that slice and return error figures, so only small
results travel back.
"""

from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np


def _init_worker(threads: int) -> None:
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(threads)
    except Exception:  # pragma: no cover - threadpoolctl missing: BLAS default
        pass


def _fwd_errors(args):
    """(bh, max |O_gpu - O_ref|, max |LSE_gpu - LSE_ref|) of one slice."""
    import oracle
    bh, q, k, v, o_gpu, lse_gpu, scale, causal, window = args
    ro, rl = oracle.attn_fwd_ref(q[None, None], k[None, None], v[None, None], scale, causal,
                                 window=window)
    eo = float(np.max(np.abs(o_gpu.astype(np.float64) - ro[0, 0])))
    el = float(np.max(np.abs(lse_gpu.astype(np.float64) - rl[0, 0])))
    return bh, eo, el


def _bwd_errors(args):
    """(bh, [(max err, max |ref|) for dQ, dK, dV]) of one slice."""
    import oracle
    bh, q, k, v, do, grads, scale, causal, window = args
    refs = oracle.attn_bwd_ref(q[None, None], k[None, None], v[None, None], do[None, None], scale,
                               causal, window=window)
    out = []
    for g, r in zip(grads, refs):
        r = r[0, 0]
        out.append((float(np.max(np.abs(g.astype(np.float64) - r))), float(np.max(np.abs(r)))))
    return bh, out


def _pool():
    cores = len(os.sched_getaffinity(0))
    workers = max(1, min(8, cores // 2))
    return cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"),
                                  initializer=_init_worker,
                                  initargs=(max(1, cores // workers),))


def _np32(t, idx):
    """Slice ``idx`` of a [B, H, ...] torch tensor as a float32 NumPy array (exact)."""
    return t[idx].float().numpy()


def fwd_errors_all_heads(x: dict, o, lse, scale: float, causal: bool, window=None):
    """Errors of every (batch, head) slice of a forward result; a list of
    (bh, O error, LSE error) sorted by bh.  ``x`` holds the host inputs, ``o`` and
    ``lse`` the GPU results (host tensors)."""
    B, H = x["q"].shape[:2]
    jobs = []
    for bh in range(B * H):
        i = divmod(bh, H)
        jobs.append((bh, _np32(x["q"], i), _np32(x["k"], i), _np32(x["v"], i), _np32(o, i),
                     lse[i].numpy().astype(np.float32), scale, causal, window))
    with _pool() as ex:
        return sorted(ex.map(_fwd_errors, jobs))


def bwd_errors_all_heads(x: dict, grads, scale: float, causal: bool, heads=None, window=None):
    """Errors of the chosen (default: every) (batch, head) slice of a backward result;
    a list of (bh, [(err, max |ref|) for dQ, dK, dV]) sorted by bh."""
    B, H = x["q"].shape[:2]
    todo = range(B * H) if heads is None else heads
    jobs = []
    for bh in todo:
        i = divmod(bh, H)
        jobs.append((bh, _np32(x["q"], i), _np32(x["k"], i), _np32(x["v"], i), _np32(x["do"], i),
                     [_np32(g, i) for g in grads], scale, causal, window))
    with _pool() as ex:
        return sorted(ex.map(_bwd_errors, jobs))
