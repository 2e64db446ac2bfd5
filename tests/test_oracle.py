"""Pins of the fp64 CPU oracle against things other than itself.

Each pin is a function of the oracle's two entry points (forward, backward), so
the same pins can be run against deliberately broken copies of the oracle
(``test_pins_catch_planted_mistakes``): every planted mistake -- a wrong causal
diagonal, a dropped scale, a dropped term of the softmax gradient, a transposed
probability matrix, a log in the wrong base -- must fail at least one pin.

What the pins rest on:
  * the scalar C brute force (independent code);
  * PyTorch's fp64 CPU attention and autograd (library routines);
  * closed forms (Q = 0, N = 1, constant V, causal row 0);
  * invariances (a common shift of all keys, a permutation of the keys);
  * central finite differences of L = sum(O * dO).
The pages say the method is exact up to rounding ("Flash Attention spiegata",
"Attention standard vs Flash attention"; "Flash Attention 2: attivarla",
"Perché Flash Attention 2"), so all of these must hold to fp64 rounding.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt
from oracle.brute import brute_bwd, brute_fwd
from exact_io_aware_74_b200.workloads import WORKLOADS, make_inputs, workload_inputs

RTOL = 1e-12


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return scale * rng.standard_normal(shape)


def _close(a, b, tol=RTOL):
    a, b = np.asarray(a), np.asarray(b)
    denom = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * denom, f"max abs err {err:.3e} > {tol:.1e} * {denom:.3e}"


def _torch_sdpa(q, k, v, scale, causal):
    tq, tk, tv = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=causal, scale=scale).numpy()


# ----------------------------------------------------------------------------------
# pins, each a function of (fwd, bwd)
# ----------------------------------------------------------------------------------

SMALL_SHAPES = [(1, 2, 1, 4), (1, 2, 5, 4), (1, 2, 33, 4), (1, 2, 33, 64), (2, 1, 17, 8)]


def pin_brute_force(fwd, bwd):
    for i, shape in enumerate(SMALL_SHAPES):
        for causal in (False, True):
            q, k, v, do = (_rand(shape, 10 * i + j) for j in range(4))
            s = 1.0 / math.sqrt(shape[-1])
            o, lse = fwd(q, k, v, s, causal)
            bo, blse = brute_fwd(q, k, v, s, causal)
            _close(o, bo)
            _close(lse, blse)
            dq, dk, dv = bwd(q, k, v, do, s, causal)
            bq, bk, bv = brute_bwd(q, k, v, do, s, causal)
            _close(dq, bq)
            _close(dk, bk)
            _close(dv, bv)


def pin_torch_library(fwd, bwd):
    threads = torch.get_num_threads()
    torch.set_num_threads(1)  # one summation order on the library side
    try:
        _pin_torch_library(fwd, bwd)
    finally:
        torch.set_num_threads(threads)


def _pin_torch_library(fwd, bwd):
    for i, (B, H, N, d) in enumerate([(2, 3, 37, 16), (1, 2, 64, 32)]):
        for causal in (False, True):
            q, k, v, do = (_rand((B, H, N, d), 100 + 4 * i + j) for j in range(4))
            s = 0.3 + 0.1 * i
            o, lse = fwd(q, k, v, s, causal)
            _close(o, _torch_sdpa(q, k, v, s, causal))
            tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
            sc = s * tq @ tk.transpose(-1, -2)
            if causal:
                sc = sc.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
            _close(lse, torch.logsumexp(sc, dim=-1).detach().numpy())
            to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                                  scale=s)
            (to * torch.from_numpy(do)).sum().backward()
            dq, dk, dv = bwd(q, k, v, do, s, causal)
            _close(dq, tq.grad.numpy(), 1e-9)
            _close(dk, tk.grad.numpy(), 1e-9)
            _close(dv, tv.grad.numpy(), 1e-9)


def pin_rows_sum_to_one(fwd, bwd):
    q, k = _rand((1, 2, 29, 8), 1), _rand((1, 2, 29, 8), 2)
    for causal in (False, True):
        p = oracle.attn_probs_ref(q, k, 0.5, causal)
        _close(p.sum(-1), np.ones((1, 2, 29)))
        if causal:
            assert np.all(np.triu(p[0, 0], 1) == 0)


def pin_constant_v(fwd, bwd):
    B, H, N, d = 1, 2, 40, 8
    q, k = _rand((B, H, N, d), 3, 3.0), _rand((B, H, N, d), 4, 3.0)
    row = _rand((d,), 5)
    v = np.broadcast_to(row, (B, H, N, d)).copy()
    for causal in (False, True):
        o, _ = fwd(q, k, v, 0.7, causal)
        _close(o, v)


def pin_causal_row0_and_n1(fwd, bwd):
    B, H, N, d = 2, 2, 9, 8
    q, k, v = (_rand((B, H, N, d), 6 + j) for j in range(3))
    s = 0.4
    o, lse = fwd(q, k, v, s, True)
    _close(o[:, :, 0], v[:, :, 0])
    _close(lse[:, :, 0], s * np.einsum("bhc,bhc->bh", q[:, :, 0], k[:, :, 0]))
    for causal in (False, True):
        o1, l1 = fwd(q[:, :, :1], k[:, :, :1], v[:, :, :1], s, causal)
        _close(o1, v[:, :, :1])
        _close(l1[:, :, 0], s * np.einsum("bhc,bhc->bh", q[:, :, 0], k[:, :, 0]))


def pin_zero_queries(fwd, bwd):
    B, H, N, d = 1, 3, 21, 8
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, H, N, d), 9), _rand((B, H, N, d), 10)
    o, lse = fwd(q, k, v, 1.3, False)
    _close(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape))
    _close(lse, np.full((B, H, N), math.log(N)))
    o, lse = fwd(q, k, v, 1.3, True)
    counts = np.arange(1, N + 1)
    _close(o, np.cumsum(v, axis=2) / counts[None, None, :, None])
    _close(lse, np.broadcast_to(np.log(counts), (B, H, N)))


def pin_key_shift(fwd, bwd):
    """K' = K + 1 u^T adds s q_i.u to every visible score of row i."""
    B, H, N, d = 1, 2, 33, 16
    q, k, v, do = (_rand((B, H, N, d), 20 + j) for j in range(4))
    u = _rand((d,), 30, 4.0)
    s = 0.25
    for causal in (False, True):
        o, lse = fwd(q, k, v, s, causal)
        o2, lse2 = fwd(q, k + u, v, s, causal)
        _close(o2, o, 1e-11)
        _close(lse2, lse + s * np.einsum("bhnc,c->bhn", q, u), 1e-11)
        # the loss does not depend on a common shift of the keys: sum_j dK_j = 0
        dq, dk, dv = bwd(q, k, v, do, s, causal)
        _close(dk.sum(axis=2), np.zeros((B, H, d)), 1e-11)
        # rows of P sum to one: sum_j dV_j = sum_i dO_i
        _close(dv.sum(axis=2), do.sum(axis=2), 1e-11)


def pin_key_permutation(fwd, bwd):
    B, H, N, d = 2, 2, 31, 8
    q, k, v, do = (_rand((B, H, N, d), 40 + j) for j in range(4))
    perm = np.random.default_rng(7).permutation(N)
    o, lse = fwd(q, k, v, 0.6, False)
    o2, lse2 = fwd(q, k[:, :, perm], v[:, :, perm], 0.6, False)
    _close(o2, o)
    _close(lse2, lse)
    _, dk, dv = bwd(q, k, v, do, 0.6, False)
    _, dk2, dv2 = bwd(q, k[:, :, perm], v[:, :, perm], do, 0.6, False)
    _close(dk2, dk[:, :, perm])
    _close(dv2, dv[:, :, perm])


def pin_finite_differences(fwd, bwd):
    eps = 1e-6
    for N, causal in ((3, False), (5, True), (5, False)):
        B, H, d = 1, 1, 4
        q, k, v, do = (_rand((B, H, N, d), 50 + N + j) for j in range(4))
        s = 0.8

        def loss(qq, kk, vv):
            o, _ = fwd(qq, kk, vv, s, causal)
            return float((o * do).sum())

        grads = bwd(q, k, v, do, s, causal)
        for which, g in enumerate(grads):
            num = np.zeros_like(g)
            args = [q, k, v]
            for idx in np.ndindex(*g.shape):
                plus = [a.copy() for a in args]
                minus = [a.copy() for a in args]
                plus[which][idx] += eps
                minus[which][idx] -= eps
                num[idx] = (loss(*plus) - loss(*minus)) / (2 * eps)
            _close(g, num, 1e-6)


PINS = [pin_brute_force, pin_torch_library, pin_rows_sum_to_one, pin_constant_v,
        pin_causal_row0_and_n1, pin_zero_queries, pin_key_shift, pin_key_permutation,
        pin_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.attn_fwd_ref, oracle.attn_bwd_ref)


# ----------------------------------------------------------------------------------
# sliding window ("Flash Attention 2: attivarla", "Modelli con attenzione a finestra
# scorrevole non standard"): row i sees its W most recent keys i-W+1 .. i
# ----------------------------------------------------------------------------------

def test_window_matches_brute_force_and_torch():
    for (B, H, N, d), W in (((1, 2, 33, 8), 5), ((2, 1, 40, 16), 1), ((1, 2, 64, 32), 17)):
        q, k, v, do = (_rand((B, H, N, d), 200 + N + W + j) for j in range(4))
        s = 0.4
        o, lse = oracle.attn_fwd_ref(q, k, v, s, True, window=W)
        bo, bl = brute_fwd(q, k, v, s, True, window=W)
        _close(o, bo)
        _close(lse, bl)
        g = oracle.attn_bwd_ref(q, k, v, do, s, True, window=W)
        bg = brute_bwd(q, k, v, do, s, True, window=W)
        for x, y in zip(g, bg):
            _close(x, y)
        # library routine with an explicit boolean mask
        i = torch.arange(N)[:, None]
        j = torch.arange(N)[None, :]
        allowed = (j <= i) & (j > i - W)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed, scale=s)
        _close(o, to.detach().numpy())
        (to * torch.from_numpy(do)).sum().backward()
        _close(g[0], tq.grad.numpy(), 1e-10)
        _close(g[1], tk.grad.numpy(), 1e-10)
        _close(g[2], tv.grad.numpy(), 1e-10)


def test_window_closed_forms():
    B, H, N, d = 1, 2, 30, 8
    q, k, v = (_rand((B, H, N, d), 230 + j) for j in range(3))
    s = 0.7
    # W = 1: every row sees only itself
    o, lse = oracle.attn_fwd_ref(q, k, v, s, True, window=1)
    _close(o, v)
    _close(lse, s * np.einsum("bhnc,bhnc->bhn", q, k))
    # W >= N: plain causal attention
    for W in (N, N + 7):
        o2, l2 = oracle.attn_fwd_ref(q, k, v, s, True, window=W)
        o3, l3 = oracle.attn_fwd_ref(q, k, v, s, True)
        _close(o2, o3)
        _close(l2, l3)
    # Q = 0: O_i is the mean of the W most recent values
    W = 4
    o, lse = oracle.attn_fwd_ref(np.zeros_like(q), k, v, 1.0, True, window=W)
    for i in range(N):
        lo = max(0, i - W + 1)
        _close(o[:, :, i], v[:, :, lo:i + 1].mean(axis=2))
        _close(lse[:, :, i], np.full((B, H), math.log(i + 1 - lo)))
    with pytest.raises(ValueError):
        oracle.attn_fwd_ref(q, k, v, s, False, window=3)


def test_window_finite_differences():
    B, H, N, d, W = 1, 1, 6, 4, 3
    q, k, v, do = (_rand((B, H, N, d), 240 + j) for j in range(4))
    s, eps = 0.9, 1e-6
    grads = oracle.attn_bwd_ref(q, k, v, do, s, True, window=W)
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            a = [q.copy(), k.copy(), v.copy()]
            b = [q.copy(), k.copy(), v.copy()]
            a[which][idx] += eps
            b[which][idx] -= eps
            fp = float((oracle.attn_fwd_ref(*a, s, True, window=W)[0] * do).sum())
            fm = float((oracle.attn_fwd_ref(*b, s, True, window=W)[0] * do).sum())
            num[idx] = (fp - fm) / (2 * eps)
        _close(g, num, 1e-6)


# ----------------------------------------------------------------------------------
# decode-like attention: Nq queries (the last positions) against Nk keys
# ----------------------------------------------------------------------------------

def test_decode_is_the_tail_of_full_causal_attention():
    """Decoding q after a prefix equals the last Nq rows of causal attention over
    [prefix; q] (both sides of the check use their own code paths)."""
    B, H, Nk, d = 2, 2, 45, 16
    for Nq in (1, 3, 45):
        k, v = _rand((B, H, Nk, d), 300 + Nq), _rand((B, H, Nk, d), 301 + Nq)
        qfull = _rand((B, H, Nk, d), 302 + Nq)
        q = qfull[:, :, Nk - Nq:]
        o, lse = oracle.attn_fwd_decode_ref(q, k, v, 0.3, True)
        fo, fl = oracle.attn_fwd_ref(qfull, k, v, 0.3, True)
        _close(o, fo[:, :, Nk - Nq:])
        _close(lse, fl[:, :, Nk - Nq:])
        # without the mask it is plain attention of those rows
        o2, l2 = oracle.attn_fwd_decode_ref(q, k, v, 0.3, False)
        fo2, fl2 = oracle.attn_fwd_ref(qfull, k, v, 0.3, False)
        _close(o2, fo2[:, :, Nk - Nq:])
        _close(l2, fl2[:, :, Nk - Nq:])


def test_decode_matches_torch_with_mask():
    B, H, Nq, Nk, d = 1, 3, 5, 70, 32
    q, k, v = _rand((B, H, Nq, d), 310), _rand((B, H, Nk, d), 311), _rand((B, H, Nk, d), 312)
    allowed = torch.arange(Nk)[None, :] <= (Nk - Nq + torch.arange(Nq)[:, None])
    to = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=allowed,
        scale=0.2)
    o, _ = oracle.attn_fwd_decode_ref(q, k, v, 0.2, True)
    _close(o, to.numpy())
    with pytest.raises(ValueError):
        oracle.attn_fwd_decode_ref(k, q, q, 0.2, True)  # Nq > Nk


# ----------------------------------------------------------------------------------
# planted mistakes (in copies of the oracle, on the CPU) must fail some pin
# ----------------------------------------------------------------------------------

def _mut_scores_diag(q_rows, k, row0, scale, causal, window=None):
    """Causal mask that also hides the diagonal (j >= i instead of j > i)."""
    n_rows = q_rows.shape[0]
    n_keys = min(k.shape[0], row0 + n_rows) if causal else k.shape[0]
    s = scale * (q_rows @ k[:n_keys].T)
    if causal:
        rows = row0 + np.arange(n_rows)[:, None]
        cols = np.arange(n_keys)[None, :]
        s = np.where(cols >= rows, -np.inf, s)
        s[:, 0] = np.where(np.isinf(s[:, 0]), 0.0, s[:, 0])  # keep row 0 finite
    return s, n_keys


def _mut_softmax_log2(s):
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return e / z, (m + np.log2(z))[:, 0]


def _bwd_variant(kind):
    def bwd(q, k, v, do, scale, causal):
        q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
        B, H, N, d = q.shape
        dq, dk, dv = (np.zeros((B, H, N, d)) for _ in range(3))
        for b in range(B):
            for h in range(H):
                s, nk = oatt._scores(q[b, h], k[b, h], 0, scale, causal)
                p, _ = oatt._softmax_rows(s)
                dp = do[b, h] @ v[b, h, :nk].T
                dd = 0.0 if kind == "drop_D" else (p * dp).sum(1, keepdims=True)
                ds = p * (dp - dd)
                ks = 1.0 if kind == "drop_dk_scale" else scale
                pv = p if kind == "transpose_dv" else p.T
                dv[b, h, :nk] = pv @ do[b, h] if kind != "transpose_dv" else (pv @ do[b, h])[:nk]
                dq[b, h] = scale * ds @ k[b, h, :nk]
                dk[b, h, :nk] = ks * ds.T @ q[b, h]
        return dq, dk, dv
    return bwd


MUTANTS = ["causal_diag", "lse_log2", "drop_D", "drop_dk_scale", "transpose_dv"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_pins_catch_planted_mistakes(mutant, monkeypatch):
    fwd, bwd = oracle.attn_fwd_ref, oracle.attn_bwd_ref
    if mutant == "causal_diag":
        monkeypatch.setattr(oatt, "_scores", _mut_scores_diag)
    elif mutant == "lse_log2":
        monkeypatch.setattr(oatt, "_softmax_rows", _mut_softmax_log2)
    else:
        bwd = _bwd_variant(mutant)
    failed = []
    for pin in PINS:
        if pin is pin_finite_differences and mutant in ("causal_diag", "lse_log2"):
            continue  # forward mutants are caught faster elsewhere
        try:
            pin(fwd, bwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"planted mistake {mutant!r} passed every pin"


def test_bwd_variant_is_exact_when_unmutated():
    """The mutant scaffold itself reproduces the oracle when nothing is planted."""
    q, k, v, do = (_rand((1, 2, 13, 8), 70 + j) for j in range(4))
    for causal in (False, True):
        a = _bwd_variant("none")(q, k, v, do, 0.5, causal)
        b = oracle.attn_bwd_ref(q, k, v, do, 0.5, causal)
        for x, y in zip(a, b):
            _close(x, y)


# ----------------------------------------------------------------------------------
# internal consistency of the oracle's own entry points
# ----------------------------------------------------------------------------------

def test_row_chunking_and_row_sampler_agree():
    q, k, v, do = (_rand((2, 2, 70, 16), 80 + j) for j in range(4))
    for causal in (False, True):
        o, lse = oracle.attn_fwd_ref(q, k, v, 0.3, causal)
        o7, lse7 = oracle.attn_fwd_ref(q, k, v, 0.3, causal, row_chunk=7)
        _close(o7, o)
        _close(lse7, lse)
        rows = [0, 1, 33, 69]
        bo, blse = brute_fwd(q, k, v, 0.3, causal)
        ro, rl = oracle.attn_fwd_rows_ref(q, k, v, 0.3, causal, bh=3, rows=rows)
        _close(ro, bo[1, 1, rows])
        _close(rl, blse[1, 1, rows])
        g = oracle.attn_bwd_ref(q, k, v, do, 0.3, causal)
        g9 = oracle.attn_bwd_ref(q, k, v, do, 0.3, causal, row_chunk=9, heads=[2])
        for x, y in zip(g9, g):
            _close(x[1, 0], y[1, 0])
            assert np.isnan(x[0, 0]).all()


def test_D_equals_rowdot_of_output():
    """D_i = sum_j P_ij dP_ij equals sum_c dO_ic O_ic (used by the GPU backward)."""
    q, k, v, do = (_rand((1, 1, 24, 8), 90 + j) for j in range(4))
    for causal in (False, True):
        o, _ = oracle.attn_fwd_ref(q, k, v, 0.5, causal)
        p = oracle.attn_probs_ref(q, k, 0.5, causal)[0, 0]
        dp = do[0, 0] @ v[0, 0].T
        _close((p * dp).sum(1), (do[0, 0] * o[0, 0]).sum(1))


# ----------------------------------------------------------------------------------
# the seeded input recipe
# ----------------------------------------------------------------------------------

def test_inputs_are_seeded_and_exact_in_fp64():
    a = make_inputs(1, 2, 64, 16, "bf16", 5, with_do=True)
    b = make_inputs(1, 2, 64, 16, "bf16", 5, with_do=True)
    for key in ("q", "k", "v", "do"):
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
        # upcast to fp64 and back is lossless
        assert torch.equal(a[key].double().to(torch.bfloat16), a[key])
    c = make_inputs(1, 2, 64, 16, "bf16", 6)
    assert not torch.equal(a["q"], c["q"])


def test_outlier_rows_recipe():
    w = WORKLOADS["fwd_bf16_b1h32_n32768_d128_causal_outliers"]
    x = make_inputs(1, 2, 1000, 8, "bf16", w.seed, outlier_frac=0.01, outlier_mult=8.0)
    plain = make_inputs(1, 2, 1000, 8, "bf16", w.seed)
    rows = x["outlier_rows"]
    assert rows.shape == (1, 2, 10)
    for h in range(2):
        idx = rows[0, h]
        assert len(set(idx.tolist())) == 10
        mask = torch.zeros(1000, dtype=torch.bool)
        mask[idx] = True
        # non-outlier rows unchanged, outlier rows exactly x8 (power of two)
        assert torch.equal(x["k"][0, h, ~mask], plain["k"][0, h, ~mask])
        assert torch.equal(x["k"][0, h, mask].float(), 8 * plain["k"][0, h, mask].float())


def test_workload_table():
    flops = {n: w.fwd_flops for n, w in WORKLOADS.items()}
    assert flops["fwd_fp16_b1h2_n128_d64"] == 4 * 2 * 128 * 128 * 64
    assert flops["fwd_bf16_b2h32_n8192_d128"] == pytest.approx(2.199e12, rel=1e-3)
    w4 = WORKLOADS["fwdbwd_bf16_b8h16_n4096_d128_causal"]
    assert w4.bwd_flops == pytest.approx(1.374e12, rel=1e-3)
    small = workload_inputs(WORKLOADS["fwd_fp16_b1h2_n128_d64"])
    assert small["q"].dtype == torch.float16 and small["q"].shape == (1, 2, 128, 64)


# ----------------------------------------------------------------------------------
# the FMA-pipe exp2 of the CUDA library (csrc/ptx.cuh, exp2_poly3), emulated in fp32
# ----------------------------------------------------------------------------------

def _exp2_poly3_f32(x):
    """Step-by-step fp32 emulation of exp2_poly3: rint range reduction + cubic."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    j = (t - f32(12582912.0)).astype(f32)
    f = (x - j).astype(f32)
    p = (f.astype(np.float64) * f32(0.055171661) + f32(0.24261114)).astype(f32)
    p = (f.astype(np.float64) * p + f32(0.69326099)).astype(f32)
    p = (f.astype(np.float64) * p + f32(0.99992807)).astype(f32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_poly3_relative_error_bound():
    x = np.concatenate([np.linspace(-124.0, 8.0, 400001), np.linspace(-1.0, 1.0, 100001)])
    got = _exp2_poly3_f32(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float32).astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4  # fitted bound 7.5e-5, below the fp16 half-ulp 2.4e-4
    assert 0 < _exp2_poly3_f32(np.array([-np.inf]))[0] < 1e-37  # clamped, not NaN


def test_window_flop_count():
    """Algorithmic FLOPs of a windowed workload: sum over rows of min(i+1, W) keys."""
    from exact_io_aware_74_b200.workloads import Workload
    w = Workload("x", 1, 1, 10, 4, "bf16", True, 0, window=3)
    pairs = sum(min(i + 1, 3) for i in range(10))
    assert w.fwd_flops == 4 * 4 * pairs
    full = Workload("y", 1, 1, 10, 4, "bf16", True, 0, window=10)
    assert full.fwd_flops == Workload("z", 1, 1, 10, 4, "bf16", True, 0).fwd_flops + 4 * 4 * 5


# ------------------------------------------------------------------------------------
# 8-bit inputs: E4M3 decoding ("Flash Attention spiegata", FlashAttention-3 section)
# ------------------------------------------------------------------------------------

def test_e4m3_decode_anchor_values():
    """Values fixed by the format: bias 7, three mantissa bits, no infinities."""
    d = oracle.e4m3_decode(np.array([0x00, 0x80, 0x01, 0x07, 0x08, 0x38, 0x39, 0x3F, 0x40,
                                     0x77, 0x7E, 0xFE, 0xB8], dtype=np.uint8))
    expect = [0.0, -0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.125, 1.875, 2.0,
              240.0, 448.0, -448.0, -1.0]
    assert np.array_equal(d, expect)
    assert np.signbit(d[1])
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(oracle.e4m3_decode(codes), ref, equal_nan=True)


def test_e4m3_decode_is_monotone_over_positive_codes():
    v = oracle.e4m3_decode(np.arange(0x00, 0x7F, dtype=np.uint8))  # 0 .. 448
    assert np.all(np.diff(v) > 0)


def test_fp8_ref_is_attention_of_the_real_values():
    """The 8-bit reference equals the scalar brute force on the decoded, scaled
    inputs (codes drawn at random, scales powers of two)."""
    from exact_io_aware_74_b200.workloads import make_fp8_inputs
    x = make_fp8_inputs(1, 2, 19, 16, seed=3)
    codes = {n: x[n].view(torch.uint8).numpy() for n in ("q", "k", "v")}
    s = x["scale"]
    for causal in (False, True):
        o, lse = oracle.attn_fwd_fp8_ref(codes["q"], codes["k"], codes["v"], 0.25, causal,
                                         s, s, 2 * s)
        real = {n: oracle.e4m3_decode(codes[n]) * (2 * s if n == "v" else s) for n in codes}
        bo, bl = brute_fwd(real["q"], real["k"], real["v"], 0.25, causal)
        _close(o, bo)
        _close(lse, bl)


def test_fp8_inputs_recipe():
    from exact_io_aware_74_b200.workloads import make_fp8_inputs
    x = make_fp8_inputs(1, 1, 64, 32, seed=11)
    assert x["q"].dtype == torch.float8_e4m3fn and x["scale"] == 1 / 16
    g = torch.Generator().manual_seed(11)
    q = torch.randn((1, 1, 64, 32), generator=g) * 16
    assert torch.equal(x["q"].view(torch.uint8), q.to(torch.float8_e4m3fn).view(torch.uint8))
    assert float(x["q"].float().abs().max()) < 448
