"""ctypes binding of libfa2.so (declared in include/fa2.h).

Argument marshalling only: every step of the attention computation runs in the
library's CUDA kernels.  Tensors are torch CUDA tensors (PyTorch provides device
memory and streams); they are passed to the C ABI as raw device pointers.  A
missing or unloadable library raises ``RuntimeError`` -- there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa2.so")

FA2_OK = 0
FA2_ERR_INVALID_ARG = 1
FA2_ERR_UNSUPPORTED = 2
FA2_ERR_ARCH = 3
FA2_ERR_CUDA = 4
FA2_ERR_TIMEOUT = 5
FA2_ERR_WORKSPACE = 6
FA2_FP16 = 0
FA2_BF16 = 1
FA2_BWD_DETERMINISTIC = 1  # flag of fa2_bwd_ex

# Every symbol include/fa2.h declares.
EXPORTS = ("fa2_fwd", "fa2_fwd_window", "fa2_fwd_fp8", "fa2_fwd_tiles_per_cta",
           "fa2_fwd_decode_splits", "fa2_fwd_decode_workspace_size", "fa2_fwd_decode",
           "fa2_bwd_workspace_size", "fa2_bwd", "fa2_bwd_window", "fa2_bwd_ex",
           "fa2_bwd_ex_workspace_size", "fa2_bwd_noalloc", "fa2_get_device_status",
           "fa2_status_string", "fa2_debug_set", "fa2_debug_set_bwd_grid",
           "fa2_debug_set_fwd_tiles", "fa2_launch_count")

_lib = None


class FA2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load() -> ctypes.CDLL:
    """Open libfa2.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m exact_io_aware_74_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa2_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    lib.fa2_fwd.restype = i
    lib.fa2_fwd_window.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    lib.fa2_fwd_window.restype = i
    lib.fa2_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, f, f, f, vp]
    lib.fa2_fwd_fp8.restype = i
    lib.fa2_fwd_tiles_per_cta.argtypes = [i, i, i, i, i, i, i]
    lib.fa2_fwd_tiles_per_cta.restype = i
    lib.fa2_fwd_decode_splits.argtypes = [i, i, i, i, i, i]
    lib.fa2_fwd_decode_splits.restype = i
    lib.fa2_fwd_decode_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.fa2_fwd_decode_workspace_size.restype = sz
    lib.fa2_fwd_decode.argtypes = [vp] * 5 + [i, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.fa2_fwd_decode.restype = i
    lib.fa2_bwd_window.argtypes = [vp] * 10 + [sz, i, i, i, i, f, i, i, vp]
    lib.fa2_bwd_window.restype = i
    lib.fa2_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa2_bwd_workspace_size.restype = sz
    lib.fa2_bwd.argtypes = [vp] * 10 + [sz, i, i, i, i, f, i, i, vp]
    lib.fa2_bwd.restype = i
    lib.fa2_bwd_ex.argtypes = [vp] * 10 + [sz, i, i, i, i, f, i, i, i, i, vp]
    lib.fa2_bwd_ex.restype = i
    lib.fa2_bwd_ex_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa2_bwd_ex_workspace_size.restype = sz
    lib.fa2_bwd_noalloc.argtypes = [vp] * 9 + [i, i, i, i, f, i, i, vp]
    lib.fa2_bwd_noalloc.restype = i
    lib.fa2_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.fa2_get_device_status.restype = i
    lib.fa2_status_string.argtypes = [i]
    lib.fa2_status_string.restype = ctypes.c_char_p
    lib.fa2_debug_set.argtypes = [i, ctypes.c_uint]
    lib.fa2_debug_set.restype = None
    lib.fa2_debug_set_bwd_grid.argtypes = [i]
    lib.fa2_debug_set_bwd_grid.restype = None
    lib.fa2_debug_set_fwd_tiles.argtypes = [i]
    lib.fa2_debug_set_fwd_tiles.restype = None
    lib.fa2_launch_count.argtypes = []
    lib.fa2_launch_count.restype = ctypes.c_ulonglong
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().fa2_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FA2_BF16
    if t.dtype == torch.float16:
        return FA2_FP16
    raise TypeError(f"unsupported dtype {t.dtype}; use float16 or bfloat16")


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check_layout(*ts):
    for t in ts:
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def fa2_fwd(q, k, v, o, lse, scale: float, causal: bool, stream=None) -> int:
    """Raw call: q, k, v, o [B,H,N,d] 16-bit; lse [B,H,N] float32.  Returns the status."""
    _check_layout(q, k, v, o, lse)
    B, H, N, d = q.shape
    return load().fa2_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                          float(scale), int(bool(causal)), _dtype_code(q), _stream(stream))


def fa2_fwd_window(q, k, v, o, lse, scale: float, window: int, stream=None) -> int:
    """Raw call of the sliding-window forward (causal, ``window`` most recent keys)."""
    _check_layout(q, k, v, o, lse)
    B, H, N, d = q.shape
    return load().fa2_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                 float(scale), int(window), _dtype_code(q), _stream(stream))


def fa2_fwd_fp8(q, k, v, o, lse, scale: float, causal: bool, q_scale: float, k_scale: float,
                v_scale: float, stream=None) -> int:
    """Raw call: q, k, v [B,H,N,d] float8_e4m3fn; o [B,H,N,d] bfloat16; lse float32."""
    _check_layout(q, k, v, o, lse)
    for t in (q, k, v):
        if t.dtype != torch.float8_e4m3fn:
            raise TypeError("q, k, v must be float8_e4m3fn")
    if o.dtype != torch.bfloat16:
        raise TypeError("o must be bfloat16")
    B, H, N, d = q.shape
    return load().fa2_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                              float(scale), int(bool(causal)), float(q_scale), float(k_scale),
                              float(v_scale), _stream(stream))


def fa2_fwd_tiles_per_cta(B: int, H: int, N: int, d: int, causal: bool, window: int = 0,
                          sm_count: int = 0) -> int:
    """Query tiles per CTA the forward uses for these sizes (1 or 2; 0 if rejected)."""
    return load().fa2_fwd_tiles_per_cta(int(B), int(H), int(N), int(d), int(bool(causal)),
                                        int(window), int(sm_count))


def fa2_fwd_decode_splits(B: int, H: int, Nq: int, Nk: int, d: int, sm_count: int = 0) -> int:
    """Split count the library picks for these sizes (0: invalid sizes or no device)."""
    return int(load().fa2_fwd_decode_splits(B, H, Nq, Nk, d, sm_count))


def fa2_fwd_decode_workspace_size(B: int, H: int, Nq: int, Nk: int, d: int,
                                  n_splits: int) -> int:
    return int(load().fa2_fwd_decode_workspace_size(B, H, Nq, Nk, d, n_splits))


def fa2_fwd_decode(q, k, v, o, lse, scale: float, causal: bool, n_splits: int, workspace,
                   stream=None) -> int:
    """Raw call: q, o [B,H,Nq,d]; k, v [B,H,Nk,d]; lse [B,H,Nq] float32;
    ``workspace`` a uint8 CUDA tensor or None.  Returns the status."""
    _check_layout(q, k, v, o, lse)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return load().fa2_fwd_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                                 float(scale), int(bool(causal)), _dtype_code(q), int(n_splits),
                                 _ptr(workspace), ws_bytes, _stream(stream))


def fa2_bwd_window(q, k, v, o, do, lse, dq, dk, dv, workspace, scale: float, window: int,
                   stream=None) -> int:
    """Raw call of the sliding-window backward."""
    _check_layout(q, k, v, o, do, lse, dq, dk, dv)
    B, H, N, d = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return load().fa2_bwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                 _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, B, H,
                                 N, d, float(scale), int(window), _dtype_code(q),
                                 _stream(stream))


def fa2_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load().fa2_bwd_workspace_size(B, H, N, d))


def fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, workspace, scale: float, causal: bool,
            stream=None) -> int:
    """Raw call; ``workspace`` is a uint8 CUDA tensor.  Returns the status."""
    _check_layout(q, k, v, o, do, lse, dq, dk, dv)
    B, H, N, d = q.shape
    ws_ptr = _ptr(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return load().fa2_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                          _ptr(dk), _ptr(dv), ws_ptr, ws_bytes, B, H, N, d, float(scale),
                          int(bool(causal)), _dtype_code(q), _stream(stream))


def fa2_bwd_ex_workspace_size(B: int, H: int, N: int, d: int, flags: int) -> int:
    return int(load().fa2_bwd_ex_workspace_size(B, H, N, d, int(flags)))


def fa2_bwd_ex(q, k, v, o, do, lse, dq, dk, dv, workspace, scale: float, causal: bool,
               window: int = 0, flags: int = 0, stream=None) -> int:
    """Raw call of the backward with options (window, FA2_BWD_DETERMINISTIC)."""
    _check_layout(q, k, v, o, do, lse, dq, dk, dv)
    B, H, N, d = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return load().fa2_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                             _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, B, H, N, d,
                             float(scale), int(bool(causal)), int(window), int(flags),
                             _dtype_code(q), _stream(stream))


def fa2_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, scale: float, causal: bool,
                    stream=None) -> int:
    """Raw call of the allocation-free backward (library-owned scratch).  Returns the status."""
    _check_layout(q, k, v, o, do, lse, dq, dk, dv)
    B, H, N, d = q.shape
    return load().fa2_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                  _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                  int(bool(causal)), _dtype_code(q), _stream(stream))


def fa2_get_device_status(stream=None) -> tuple[int, int]:
    """(status, wait site) of the current device; synchronises ``stream``."""
    site = ctypes.c_int(0)
    rc = load().fa2_get_device_status(_stream(stream), ctypes.byref(site))
    return rc, site.value


def fa2_debug_set(fault: int, wait_limit_ms: int = 0) -> None:
    load().fa2_debug_set(int(fault), int(wait_limit_ms))


def fa2_debug_set_bwd_grid(max_ctas: int) -> None:
    """Test hook: cap the backward's persistent grid (0 = one CTA per SM)."""
    load().fa2_debug_set_bwd_grid(int(max_ctas))


def fa2_debug_set_fwd_tiles(tiles: int) -> None:
    """Test hook: force 1 or 2 query tiles per forward CTA (0 = the library's choice)."""
    load().fa2_debug_set_fwd_tiles(int(tiles))


def fa2_launch_count() -> int:
    return int(load().fa2_launch_count())


# ------------------------------------------------------------------------------------
# allocating conveniences (PyTorch owns the memory)
# ------------------------------------------------------------------------------------

def forward(q, k, v, scale: float, causal: bool, stream=None):
    """Allocates O and LSE, calls fa2_fwd, raises FA2Error on a bad status."""
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = fa2_fwd(q, k, v, o, lse, scale, causal, stream)
    if rc != FA2_OK:
        raise FA2Error(rc, "fa2_fwd")
    return o, lse


def forward_fp8(q, k, v, scale: float, causal: bool, q_scale: float, k_scale: float,
                v_scale: float, stream=None):
    """Allocating wrapper of fa2_fwd_fp8: bf16 O and float32 LSE."""
    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = fa2_fwd_fp8(q, k, v, o, lse, scale, causal, q_scale, k_scale, v_scale, stream)
    if rc != FA2_OK:
        raise FA2Error(rc, "fa2_fwd_fp8")
    return o, lse


def forward_window(q, k, v, scale: float, window: int, stream=None):
    """Allocating wrapper of fa2_fwd_window."""
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = fa2_fwd_window(q, k, v, o, lse, scale, window, stream)
    if rc != FA2_OK:
        raise FA2Error(rc, "fa2_fwd_window")
    return o, lse


def forward_decode(q, k, v, scale: float, causal: bool, n_splits: int = 0, stream=None):
    """Allocating wrapper of fa2_fwd_decode: q [B,H,Nq,d] against k, v [B,H,Nk,d].

    ``n_splits`` = 0 takes the library's choice for the current device.
    """
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if n_splits == 0:
        n_splits = fa2_fwd_decode_splits(B, H, Nq, Nk, d)
        if n_splits == 0:
            raise FA2Error(FA2_ERR_INVALID_ARG, "fa2_fwd_decode_splits")
    ws = fa2_fwd_decode_workspace_size(B, H, Nq, Nk, d, n_splits)
    workspace = torch.empty(ws, dtype=torch.uint8, device=q.device) if ws else None
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    rc = fa2_fwd_decode(q, k, v, o, lse, scale, causal, n_splits, workspace, stream)
    if rc != FA2_OK:
        raise FA2Error(rc, "fa2_fwd_decode")
    return o, lse


def backward_window(q, k, v, o, do, lse, scale: float, window: int, stream=None):
    """Allocating wrapper of fa2_bwd_window."""
    B, H, N, d = q.shape
    workspace = torch.empty(fa2_bwd_workspace_size(B, H, N, d), dtype=torch.uint8,
                            device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = fa2_bwd_window(q, k, v, o, do, lse, dq, dk, dv, workspace, scale, window, stream)
    if rc != FA2_OK:
        raise FA2Error(rc, "fa2_bwd_window")
    return dq, dk, dv


def backward(q, k, v, o, do, lse, scale: float, causal: bool, workspace=None, stream=None,
             deterministic: bool = False, window: int = 0):
    """Allocates dQ, dK, dV (and the workspace if not given), calls fa2_bwd, or
    fa2_bwd_ex when ``deterministic`` or a ``window`` is asked for."""
    B, H, N, d = q.shape
    flags = FA2_BWD_DETERMINISTIC if deterministic else 0
    if workspace is None:
        workspace = torch.empty(fa2_bwd_ex_workspace_size(B, H, N, d, flags), dtype=torch.uint8,
                                device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if flags or window:
        rc = fa2_bwd_ex(q, k, v, o, do, lse, dq, dk, dv, workspace, scale, causal, window, flags,
                        stream)
        where = "fa2_bwd_ex"
    else:
        rc = fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, workspace, scale, causal, stream)
        where = "fa2_bwd"
    if rc != FA2_OK:
        raise FA2Error(rc, where)
    return dq, dk, dv
