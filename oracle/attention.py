"""fp64 NumPy oracle: the plain definition of softmax attention and its gradient.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Arrays are [B, H, N, d] (queries, keys, values, output, output gradient) and
[B, H, N] (log-sum-exp).  Inputs may be any real dtype; they are upcast exactly
to float64 before any arithmetic, so the oracle sees precisely the 16-bit values
the GPU sees.  Per (batch, head) slice the full score rows are materialised for a
chunk of query rows (memory is chunk x N, never N x N for large N), the softmax
of each row is taken exactly (subtract the row maximum, exponentiate, divide by
the sum) and the rest are ordinary matrix products.  Nothing here is tiled over
keys or computed incrementally: that is the GPU path's business, and the point
of this module is to be the reference it is checked against.

Sources (page title, section):
  * "Flash Attention spiegata: una guida completa" (datacamp), "Attention
    standard vs Flash attention": the fast method computes exactly standard
    attention.
  * "FlashAttention-2" (systems-analysis.info wiki), "Предпосылки": standard
    attention materialises the full score matrix -- which is what this oracle
    does, a chunk of rows at a time.
  * "Flash Attention spiegata", "Ricomputazione": the backward pass recomputes
    the probabilities from the scores; here they are recomputed from scratch
    per chunk as well.
"""

from __future__ import annotations

import numpy as np

_ROW_CHUNK = 1024


def _f64(x) -> np.ndarray:
    """Exact upcast to float64 (torch tensors are converted through numpy)."""
    if hasattr(x, "detach"):  # torch.Tensor without importing torch here
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _check_shapes(q, k, v):
    if q.ndim != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B, H, N, d] with equal shapes")


def _scores(q_rows: np.ndarray, k: np.ndarray, row0: int, scale: float,
            causal: bool, window: int | None = None) -> tuple[np.ndarray, int]:
    """Scaled scores S = scale * q_rows k^T for query rows row0..row0+len-1.

    With ``causal`` the keys after each row's own position are set to -inf and
    only keys 0..row_last are formed at all.  With a sliding ``window`` W (causal
    only) row i also loses the keys before i - W + 1, so that it sees the W most
    recent keys (itself included).  Returns (S, number of keys used).
    """
    n_rows = q_rows.shape[0]
    n_keys = min(k.shape[0], row0 + n_rows) if causal else k.shape[0]
    s = scale * (q_rows @ k[:n_keys].T)
    if causal:
        rows = row0 + np.arange(n_rows)[:, None]
        cols = np.arange(n_keys)[None, :]
        s = np.where(cols > rows, -np.inf, s)
        if window is not None:
            s = np.where(cols < rows - window + 1, -np.inf, s)
    return s, n_keys


def _check_window(causal: bool, window) -> None:
    if window is not None and (not causal or int(window) < 1):
        raise ValueError("a sliding window needs causal=True and window >= 1")


def _softmax_rows(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Exact row softmax and row log-sum-exp of a score block (fp64)."""
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return e / z, (m + np.log(z))[:, 0]


def attn_fwd_rows_ref(q, k, v, scale: float, causal: bool, bh: int,
                      rows, window: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """O and LSE of selected query rows of one flattened (batch*head) slice.

    ``q, k, v`` are [B, H, N, d]; ``bh`` indexes the flattened B*H axis; ``rows``
    is a sequence of query row indices.  Returns (O [len(rows), d],
    LSE [len(rows)]), fp64.  Used to check full-size GPU runs on a sample of
    rows without forming every row.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check_shapes(q, k, v)
    _check_window(causal, window)
    B, H, N, d = q.shape
    b, h = divmod(int(bh), H)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, d))
    lse = np.empty(rows.size)
    for t, r in enumerate(rows):
        s, nk = _scores(q[b, h, r:r + 1], k[b, h], int(r), scale, causal, window)
        p, l = _softmax_rows(s)
        out[t] = (p @ v[b, h, :nk])[0]
        lse[t] = l[0]
    return out, lse


def attn_fwd_ref(q, k, v, scale: float, causal: bool,
                 row_chunk: int = _ROW_CHUNK,
                 window: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Forward attention: O = softmax(scale * Q K^T [causal mask]) V, and LSE.

    ``window`` (causal only) restricts row i to its W most recent keys, the
    sliding-window attention of "Flash Attention 2: attivarla (llama.cpp,
    Ollama, vLLM)", section "Modelli con attenzione a finestra scorrevole non
    standard".  Returns (O [B,H,N,d], LSE [B,H,N]) in fp64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check_shapes(q, k, v)
    _check_window(causal, window)
    B, H, N, d = q.shape
    out = np.empty((B, H, N, d))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, row_chunk):
                r1 = min(N, r0 + row_chunk)
                s, nk = _scores(q[b, h, r0:r1], k[b, h], r0, scale, causal, window)
                p, l = _softmax_rows(s)
                out[b, h, r0:r1] = p @ v[b, h, :nk]
                lse[b, h, r0:r1] = l
    return out, lse


def attn_probs_ref(q, k, scale: float, causal: bool, window: int | None = None) -> np.ndarray:
    """The full probability matrix P [B,H,N,N] (tiny shapes only; for pins)."""
    _check_window(causal, window)
    q, k = _f64(q), _f64(k)
    B, H, N, d = q.shape
    p_all = np.zeros((B, H, N, N))
    for b in range(B):
        for h in range(H):
            s, nk = _scores(q[b, h], k[b, h], 0, scale, causal, window)
            p, _ = _softmax_rows(s)
            p_all[b, h, :, :nk] = p
    return p_all


def attn_bwd_ref(q, k, v, do, scale: float, causal: bool,
                 row_chunk: int = _ROW_CHUNK, heads=None, window: int | None = None):
    """Gradients of L = sum(O * dO) with respect to Q, K and V (fp64).

    The probabilities are recomputed from the scores of each chunk of query
    rows; D_i = sum_j P_ij dP_ij is taken from P and dP directly (not from the
    forward output).  ``heads`` optionally restricts the work to a list of
    flattened (batch*head) indices; other slices of the results are left as
    NaN.  Returns (dQ, dK, dV), each [B,H,N,d].
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    _check_shapes(q, k, v)
    _check_window(causal, window)
    if do.shape != q.shape:
        raise ValueError("do must have the shape of q")
    B, H, N, d = q.shape
    dq = np.full((B, H, N, d), np.nan)
    dk = np.full((B, H, N, d), np.nan)
    dv = np.full((B, H, N, d), np.nan)
    todo = range(B * H) if heads is None else [int(x) for x in heads]
    for bh in todo:
        b, h = divmod(bh, H)
        dk_bh = np.zeros((N, d))
        dv_bh = np.zeros((N, d))
        for r0 in range(0, N, row_chunk):
            r1 = min(N, r0 + row_chunk)
            s, nk = _scores(q[b, h, r0:r1], k[b, h], r0, scale, causal, window)
            p, _ = _softmax_rows(s)
            do_c = do[b, h, r0:r1]
            dv_bh[:nk] += p.T @ do_c
            dp = do_c @ v[b, h, :nk].T
            dd = (p * dp).sum(axis=1, keepdims=True)
            ds = p * (dp - dd)
            dq[b, h, r0:r1] = scale * (ds @ k[b, h, :nk])
            dk_bh[:nk] += scale * (ds.T @ q[b, h, r0:r1])
        dk[b, h] = dk_bh
        dv[b, h] = dv_bh
    return dq, dk, dv


def attn_fwd_decode_ref(q, k, v, scale: float, causal: bool) -> tuple[np.ndarray, np.ndarray]:
    """Attention of Nq queries against Nk keys (Nq <= Nk): the decode-like case.

    q is [B,H,Nq,d]; k, v are [B,H,Nk,d].  The queries are the last Nq positions
    of the sequence, so with ``causal`` query i sees keys 0 .. Nk - Nq + i
    (bottom-right alignment); without it every key.  This is the inference
    setting of "Flash Attention spiegata: una guida completa", section
    "Parallelismo lungo la lunghezza della sequenza" (small batches, long
    prompts).  Returns (O [B,H,Nq,d], LSE [B,H,Nq]) in fp64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or k.ndim != 4 or v.shape != k.shape or q.shape[:2] != k.shape[:2] \
            or q.shape[3] != k.shape[3] or q.shape[2] > k.shape[2]:
        raise ValueError("q [B,H,Nq,d] and k, v [B,H,Nk,d] with Nq <= Nk")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    out = np.empty((B, H, Nq, d))
    lse = np.empty((B, H, Nq))
    rows = (Nk - Nq) + np.arange(Nq)[:, None]
    cols = np.arange(Nk)[None, :]
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(cols > rows, -np.inf, s)
            p, l = _softmax_rows(s)
            out[b, h] = p @ v[b, h]
            lse[b, h] = l
    return out, lse


def e4m3_decode(codes) -> np.ndarray:
    """Real values of E4M3 bytes (uint8 array), from the format's definition.

    One sign bit, four exponent bits with bias 7 and three mantissa bits:
    exponent 0 holds subnormals m/8 * 2^-6; otherwise (1 + m/8) * 2^(e - 7);
    the pattern with every exponent and mantissa bit set is NaN (there are no
    infinities, so the largest finite magnitude is 1.75 * 2^8 = 448).  This is
    the 8-bit floating point that "Flash Attention spiegata: una guida
    completa", FlashAttention-3 section, names for FP8 attention.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def attn_fwd_fp8_ref(q8, k8, v8, scale: float, causal: bool, q_scale: float, k_scale: float,
                     v_scale: float) -> tuple[np.ndarray, np.ndarray]:
    """Attention of E4M3 inputs: the plain definition applied to their real values
    q_scale * Q, k_scale * K, v_scale * V (q8, k8, v8: uint8 codes [B,H,N,d]).
    Returns (O, LSE) in fp64."""
    q = e4m3_decode(q8) * q_scale
    k = e4m3_decode(k8) * k_scale
    v = e4m3_decode(v8) * v_scale
    return attn_fwd_ref(q, k, v, scale, causal)
