"""ctypes loader for the scalar C brute force in ``brute.c``.

TEST INFRASTRUCTURE ONLY: the product path never imports this module.

``build_brute()`` compiles ``brute.c`` with the host C compiler into
``oracle/_build/libbrute.so`` (the build step of ``__graft_entry__.build()`` calls
it too).  ``brute_fwd`` / ``brute_bwd`` loop over the (batch, head) slices of
[B,H,N,d] arrays and call the C routines slice by slice.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "brute.c")
_LIB = os.path.join(_HERE, "_build", "libbrute.so")
_lib = None


def build_brute(force: bool = False) -> str:
    """Compile brute.c into a shared library if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"],
                       check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_brute())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.brute_attn_fwd.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_int]
        lib.brute_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_int]
        lib.brute_set_window.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def brute_fwd(q, k, v, scale: float, causal: bool, window: int | None = None):
    """(O, LSE) of [B,H,N,d] inputs by scalar triple loops, fp64."""
    lib = _load()
    lib.brute_set_window(int(window) if window else 0)
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    o = np.zeros((B, H, N, d))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            qs, ks, vs = (np.ascontiguousarray(t[b, h]) for t in (q, k, v))
            os_ = np.zeros((N, d))
            ls = np.zeros(N)
            lib.brute_attn_fwd(_ptr(qs), _ptr(ks), _ptr(vs), _ptr(os_), _ptr(ls), N, d,
                               float(scale), int(bool(causal)))
            o[b, h], lse[b, h] = os_, ls
    return o, lse


def brute_bwd(q, k, v, do, scale: float, causal: bool, window: int | None = None):
    """(dQ, dK, dV) of [B,H,N,d] inputs by scalar loops, fp64."""
    lib = _load()
    lib.brute_set_window(int(window) if window else 0)
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    dq, dk, dv = (np.zeros((B, H, N, d)) for _ in range(3))
    for b in range(B):
        for h in range(H):
            qs, ks, vs, dos = (np.ascontiguousarray(t[b, h]) for t in (q, k, v, do))
            a, bb, c = np.zeros((N, d)), np.zeros((N, d)), np.zeros((N, d))
            lib.brute_attn_bwd(_ptr(qs), _ptr(ks), _ptr(vs), _ptr(dos), _ptr(a), _ptr(bb),
                               _ptr(c), N, d, float(scale), int(bool(causal)))
            dq[b, h], dk[b, h], dv[b, h] = a, bb, c
    return dq, dk, dv
