"""Host-side checks of the C ABI that need no GPU.

The library must load and export every symbol include/fa2.h declares, and argument
validation must reject bad calls before any CUDA call is made (so these run on a
machine without a GPU).
"""

import ctypes
import os
import re

import pytest

from exact_io_aware_74_b200 import fa2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "fa2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa2_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_74_b200 import build
    build.build()
    return fa2.load()


def test_header_declarations_match_binding():
    assert _header_functions() == sorted(fa2.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _header_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert fa2.status_string(fa2.FA2_OK) == "FA2_OK"
    assert fa2.status_string(fa2.FA2_ERR_TIMEOUT) == "FA2_ERR_TIMEOUT"
    assert fa2.status_string(99) == "FA2_ERR_UNKNOWN"


P = 1 << 20  # a fake, 16-byte aligned "device pointer": never dereferenced on these paths


@pytest.mark.parametrize("args,expect", [
    ((0, P, P, P, P, 1, 1, 64, 64, 0.1, 0, 1), fa2.FA2_ERR_INVALID_ARG),        # null Q
    ((P + 2, P, P, 2 * P, 3 * P, 1, 1, 64, 64, 0.1, 0, 1), fa2.FA2_ERR_INVALID_ARG),  # misaligned
    ((P, P, P, 2 * P, 3 * P, 0, 1, 64, 64, 0.1, 0, 1), fa2.FA2_ERR_INVALID_ARG),  # B = 0
    ((P, P, P, 2 * P, 3 * P, 1, 1, 0, 64, 0.1, 0, 1), fa2.FA2_ERR_INVALID_ARG),   # N = 0
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 64, 0.1, 2, 1), fa2.FA2_ERR_INVALID_ARG),  # causal = 2
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 64, 0.1, 0, 5), fa2.FA2_ERR_INVALID_ARG),  # dtype
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 64, float("nan"), 0, 1), fa2.FA2_ERR_INVALID_ARG),
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 64, -0.5, 0, 1), fa2.FA2_ERR_INVALID_ARG),  # scale <= 0
    ((P, P, P, P, 3 * P, 1, 1, 64, 64, 0.1, 0, 1), fa2.FA2_ERR_INVALID_ARG),     # O aliases Q
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 100, 0.1, 0, 1), fa2.FA2_ERR_UNSUPPORTED),  # d % 8 != 0
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 264, 0.1, 0, 1), fa2.FA2_ERR_UNSUPPORTED),  # d > 256
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 0, 0.1, 0, 1), fa2.FA2_ERR_UNSUPPORTED),
    ((P, P, P, 2 * P, 3 * P, 1, 1, 64, 4, 0.1, 0, 1), fa2.FA2_ERR_UNSUPPORTED),
])
def test_fwd_validation_without_device(lib, args, expect):
    assert lib.fa2_fwd(*args, None) == expect


def test_fwd_overlap_checks_use_each_buffer_size(lib):
    """An LSE buffer placed right below O (or right after it) is not an alias."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("these fake pointers are only safe without a device")
    B, H, N, d = 1, 2, 64, 64
    o_bytes, lse_bytes = B * H * N * d * 2, B * H * N * 4
    O = 64 * P
    for lse in (O - lse_bytes, O + o_bytes):
        rc = lib.fa2_fwd(P, 2 * P, 3 * P, O, lse, B, H, N, d, 0.1, 0, 1, None)
        assert rc in (fa2.FA2_ERR_CUDA, fa2.FA2_ERR_ARCH)  # validation passed
    rc = lib.fa2_fwd(P, 2 * P, 3 * P, O, O + 16, B, H, N, d, 0.1, 0, 1, None)
    assert rc == fa2.FA2_ERR_INVALID_ARG


def test_bwd_validation_without_device(lib):
    ws = fa2.fa2_bwd_workspace_size(2, 3, 1000, 128)
    assert ws > 0 and ws % 256 == 0
    # D and LSE*log2(e) padded to 128 rows per head, the 256-byte tile counter, then
    # the fp32 dQ accumulator, as wide as the kernel's tile (64 or 128 columns)
    assert ws == 2 * 2 * 3 * 1024 * 4 + 256 + 2 * 3 * 1000 * 128 * 4
    assert fa2.fa2_bwd_workspace_size(2, 3, 1000, 64) == 2 * 2 * 3 * 1024 * 4 + 256 + 2 * 3 * 1000 * 64 * 4
    # the deterministic mode keeps the two row statistics and the counter only
    assert fa2.fa2_bwd_ex_workspace_size(2, 3, 1000, 128, fa2.FA2_BWD_DETERMINISTIC) == 2 * 2 * 3 * 1024 * 4 + 256
    assert fa2.fa2_bwd_ex_workspace_size(2, 3, 1000, 64, fa2.FA2_BWD_DETERMINISTIC) == 2 * 2 * 3 * 1024 * 4 + 256
    assert fa2.fa2_bwd_ex_workspace_size(2, 3, 1000, 128, 0) == ws
    assert fa2.fa2_bwd_ex_workspace_size(2, 3, 1000, 128, 2) == 0  # unknown flag
    assert fa2.fa2_bwd_workspace_size(2, 3, 1000, 100) == 0  # d % 8 != 0
    assert fa2.fa2_bwd_workspace_size(2, 3, 1000, 136) == 0  # backward head dims end at 128
    # d = 96 runs on 128-wide tiles
    assert fa2.fa2_bwd_workspace_size(2, 3, 1000, 96) == fa2.fa2_bwd_workspace_size(2, 3, 1000, 128)
    assert fa2.fa2_bwd_workspace_size(2, 3, 1000, 8) == fa2.fa2_bwd_workspace_size(2, 3, 1000, 64)
    ptrs = [P * (i + 1) for i in range(9)]
    # workspace too small
    rc = lib.fa2_bwd(*ptrs, 16 * P, 256, 1, 1, 64, 64, 0.1, 0, 1, None)
    assert rc == fa2.FA2_ERR_WORKSPACE
    # null dK
    bad = list(ptrs)
    bad[7] = 0
    assert lib.fa2_bwd(*bad, 16 * P, ws, 1, 1, 64, 64, 0.1, 0, 1, None) == fa2.FA2_ERR_INVALID_ARG
    # dQ aliasing Q
    bad = list(ptrs)
    bad[6] = bad[0]
    assert lib.fa2_bwd(*bad, 16 * P, ws, 1, 1, 64, 64, 0.1, 0, 1, None) == fa2.FA2_ERR_INVALID_ARG


def test_device_calls_fail_cleanly_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = lib.fa2_fwd(P, 2 * P, 3 * P, 4 * P, 5 * P, 1, 1, 64, 64, 0.1, 0, 1, None)
    assert rc in (fa2.FA2_ERR_CUDA, fa2.FA2_ERR_ARCH)
    site = ctypes.c_int(7)
    assert lib.fa2_get_device_status(None, ctypes.byref(site)) == fa2.FA2_ERR_CUDA


def test_binding_fails_loudly_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(fa2, "_lib", None)
    monkeypatch.setattr(fa2, "LIB_PATH", str(tmp_path / "libfa2.so"))
    with pytest.raises(RuntimeError, match="missing"):
        fa2.load()


def test_window_validation_without_device(lib):
    args = (P, 2 * P, 3 * P, 4 * P, 5 * P, 1, 1, 64, 64, 0.1)
    assert lib.fa2_fwd_window(*args, 0, 1, None) == fa2.FA2_ERR_INVALID_ARG
    assert lib.fa2_fwd_window(*args, -5, 1, None) == fa2.FA2_ERR_INVALID_ARG
    assert lib.fa2_fwd_window(*args[:8], 100, 0.1, 8, 1, None) == fa2.FA2_ERR_UNSUPPORTED
    ptrs = [P * (i + 1) for i in range(9)]
    ws = fa2.fa2_bwd_workspace_size(1, 1, 64, 64)
    assert lib.fa2_bwd_window(*ptrs, 16 * P, ws, 1, 1, 64, 64, 0.1, 0, 1, None) == fa2.FA2_ERR_INVALID_ARG


def _decode(lib, *, q=P, k=2 * P, v=3 * P, o=4 * P, lse=5 * P, B=1, H=1, Nq=1, Nk=1000, d=64,
            scale=0.1, causal=1, dtype=1, splits=1, ws=None, ws_bytes=0):
    return lib.fa2_fwd_decode(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, splits, ws,
                              ws_bytes, None)


def test_decode_validation_without_device(lib):
    E = fa2.FA2_ERR_INVALID_ARG
    assert _decode(lib, q=0) == E
    assert _decode(lib, Nq=0) == E
    assert _decode(lib, Nq=1001) == E            # more queries than keys
    assert _decode(lib, splits=0) == E
    assert _decode(lib, splits=1025) == E
    assert _decode(lib, causal=3) == E
    assert _decode(lib, o=P) == E                 # O aliases Q
    assert _decode(lib, d=100) == fa2.FA2_ERR_UNSUPPORTED
    assert _decode(lib, d=264) == fa2.FA2_ERR_UNSUPPORTED
    # 100 queries, 1000 keys = 8 key tiles: 3 splits need a workspace
    assert _decode(lib, Nq=100, splits=3) == fa2.FA2_ERR_WORKSPACE
    need = fa2.fa2_fwd_decode_workspace_size(1, 1, 100, 1000, 64, 3)
    assert _decode(lib, Nq=100, splits=3, ws=64 * P, ws_bytes=need - 1) == fa2.FA2_ERR_WORKSPACE
    assert _decode(lib, Nq=100, splits=3, ws=64 * P + 16, ws_bytes=need) == fa2.FA2_ERR_WORKSPACE
    # a workspace that overlaps K
    assert _decode(lib, Nq=100, splits=3, ws=2 * P, ws_bytes=need) == fa2.FA2_ERR_WORKSPACE
    # up to 64 queries are replicated across the tile: partials even with one split
    assert _decode(lib, Nq=1, splits=1) == fa2.FA2_ERR_WORKSPACE


def test_decode_calls_pass_validation_then_need_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("these fake pointers are only safe without a device")
    assert _decode(lib, Nq=100) in (fa2.FA2_ERR_CUDA, fa2.FA2_ERR_ARCH)
    need = fa2.fa2_fwd_decode_workspace_size(1, 1, 1, 1000, 64, 3)
    assert _decode(lib, splits=3, ws=64 * P, ws_bytes=need) in (fa2.FA2_ERR_CUDA,
                                                                  fa2.FA2_ERR_ARCH)
    assert fa2.fa2_fwd_decode_splits(1, 32, 1, 32768, 128, 0) == 0  # no device to ask


def test_decode_workspace_size(lib):
    ws = fa2.fa2_fwd_decode_workspace_size
    # 100 queries (no copies): 1000 keys = 8 tiles; 3 splits of 3, 3, 2 tiles:
    # O part 3*100*64*4 = 76800 bytes (256-aligned), LSE part 1200 -> 1280.
    assert ws(1, 1, 100, 1000, 64, 3) == 76800 + 1280
    # 5 splits -> 2 tiles each -> 4 stretches; 100 splits -> 8 stretches of one tile
    assert ws(1, 1, 100, 1000, 64, 5) == 4 * 25600 + 1792
    assert ws(1, 1, 100, 1000, 64, 100) == 8 * 25600 + 3328
    # One split of more than 64 queries needs none.
    assert ws(1, 32, 100, 32768, 128, 1) == 0
    # One query: 4 copies per stretch.  9 stretches x 4 copies x 32 heads:
    # O part 36*32*128*4 = 589824, LSE part 36*32*4 = 4608.
    assert ws(1, 32, 1, 32768, 128, 9) == 589824 + 4608
    assert ws(1, 32, 1, 32768, 128, 1) == 4 * 32 * 512 + 512
    # 40 queries: 2 copies; one key tile, so 7 splits are one stretch:
    # O part 2*4*40*64*4 = 81920, LSE part 2*4*40*4 = 1280.
    assert ws(2, 2, 40, 128, 64, 7) == 81920 + 1280
    assert ws(1, 1, 2, 1, 64, 2) == 0       # Nq > Nk
    assert ws(1, 1, 1, 1000, 64, 0) == 0    # no split count


@pytest.mark.parametrize("shape,expect", [
    # 32 CTAs per split on 148 SMs: 4 splits fill one wave (128 CTAs).
    ((1, 32, 1, 32768, 128), 4),
    # 256 CTAs already exceed one wave.
    ((8, 32, 1, 8192, 128), 1),
    # A full prefill fills the GPU many times over.
    ((8, 16, 4096, 4096, 128), 1),
    # One head: 148 would fit, but 256 key tiles allow 64 splits of 4.
    ((1, 1, 1, 32768, 64), 64),
    # 300 queries = 2 CTAs per head per split; 8 heads: 9 splits (144 CTAs).
    ((1, 8, 300, 65536, 128), 9),
    # Fewer than 8 key tiles: nothing to split.
    ((1, 1, 1, 700, 64), 1),
])
def test_decode_split_choice(lib, shape, expect):
    assert fa2.fa2_fwd_decode_splits(*shape, 148) == expect


def test_head_dims_pick_tile_widths(lib):
    """Head dims up to 256 in multiples of 8: the decode partials are padded to the
    tile width (64, 128, 192 or 256 columns), and above 128 a CTA holds one
    128-row query tile, so a split has twice the CTAs."""
    ws = fa2.fa2_fwd_decode_workspace_size
    for d, tile in ((8, 64), (64, 64), (72, 128), (128, 128), (136, 192), (192, 192),
                    (200, 256), (256, 256)):
        assert ws(1, 1, 100, 1000, d, 2) == 2 * 100 * tile * 4 + 1024, d
    # 300 queries: 2 CTAs per head per split at d <= 128, 3 above
    assert fa2.fa2_fwd_decode_splits(1, 8, 300, 65536, 128, 148) == 9
    assert fa2.fa2_fwd_decode_splits(1, 8, 300, 65536, 256, 148) == 6


def test_bwd_rejects_head_dims_above_128(lib):
    ptrs = [P * (i + 1) for i in range(9)]
    assert lib.fa2_bwd(*ptrs, 16 * P, 1 << 30, 1, 1, 64, 192, 0.1, 0, 1, None) == \
        fa2.FA2_ERR_UNSUPPORTED


def test_decode_split_choice_rejects_bad_sizes(lib):
    assert fa2.fa2_fwd_decode_splits(1, 1, 5, 4, 64, 148) == 0
    assert fa2.fa2_fwd_decode_splits(1, 1, 1, 4, 84, 148) == 0


def test_fp8_validation_without_device(lib):
    def call(q=P, o=4 * P, N=64, d=64, scale=0.1, causal=0, qs=1.0, ks=1.0, vs=1.0):
        return lib.fa2_fwd_fp8(q, 2 * P, 3 * P, o, 5 * P, 1, 1, N, d, scale, causal, qs, ks, vs,
                               None)
    E = fa2.FA2_ERR_INVALID_ARG
    assert call(q=0) == E
    assert call(causal=2) == E
    assert call(qs=0.0) == E
    assert call(vs=float("inf")) == E
    assert call(ks=-1.0) == E
    assert call(scale=float("nan")) == E
    assert call(o=P) == E                       # O overlaps Q
    for d in (8, 24, 100, 144, 256):
        assert call(d=d) == fa2.FA2_ERR_UNSUPPORTED, d
    import torch
    if not torch.cuda.is_available():
        for d in (16, 64, 128):
            assert call(d=d) in (fa2.FA2_ERR_CUDA, fa2.FA2_ERR_ARCH)


@pytest.mark.parametrize("shape,causal,window,expect", [
    # causal, two-tile grid under one wave (16 heads x 8 blocks = 128 CTAs): one tile
    ((1, 16, 2048, 64), True, 0, 1),
    ((1, 8, 4096, 128), True, 0, 1),
    # the bench workload (4 x 16 x 4 = 256 two-tile CTAs): two
    ((4, 16, 1024, 64), True, 0, 2),
    # not causal: 128 equal two-tile CTAs; one tile would need 256 > 148: two
    ((1, 32, 1024, 64), False, 0, 2),
    # not causal, the one-tile grid fits in one wave (2 x 4 x ... = 16 / 64 CTAs): one
    ((1, 2, 1024, 64), False, 0, 1),
    ((1, 4, 2048, 128), False, 0, 1),
    # a sliding window makes the items equal: the one-wave rule for one tile
    ((1, 16, 2048, 64), True, 512, 2),
    ((1, 4, 2048, 64), True, 512, 1),
    # a window as long as the sequence is plain causal
    ((1, 16, 2048, 64), True, 4096, 1),
    # head dims above 128 always run one tile per CTA
    ((8, 16, 4096, 256), True, 0, 1),
    # the headline shape fills the GPU many times over
    ((2, 32, 8192, 128), False, 0, 2),
])
def test_forward_tiles_per_cta_choice(lib, shape, causal, window, expect):
    assert fa2.fa2_fwd_tiles_per_cta(*shape, causal, window, 148) == expect


def test_forward_tiles_per_cta_rejects_bad_sizes(lib):
    assert fa2.fa2_fwd_tiles_per_cta(1, 2, 128, 60, True, 0, 148) == 0   # d not a multiple of 8
    assert fa2.fa2_fwd_tiles_per_cta(0, 2, 128, 64, True, 0, 148) == 0   # B < 1
    assert fa2.fa2_fwd_tiles_per_cta(1, 2, 128, 64, True, -1, 148) == 0  # negative window
    assert fa2.fa2_fwd_tiles_per_cta(1, 2, 128, 64, True, 0, 0) == 0     # no device to ask


# ------------------------------------------------------------------ memory linear in N
#
# "FlashAttention-2" (systems-analysis.info wiki), "Предпосылки": the tiled method
# needs memory linear in the sequence length, because no N x N matrix is stored.
# The forward takes no scratch at all; the backward's scratch is two float rows per
# query (D and LSE * log2 e, padded to 128 rows), a 256-byte tile counter and a float
# dQ accumulator of one row per query, as wide as the kernel's tile (64 or 128
# columns); the deterministic mode, which sums dQ in tensor memory, needs the rows and
# the counter alone.

@pytest.mark.parametrize("d", [32, 64, 96, 128])
def test_bwd_workspace_is_linear_in_sequence_length(lib, d):
    B, H = 2, 3
    tile = 64 if d <= 64 else 128
    for N in (128, 1024, 4096, 32768):
        ws = lib.fa2_bwd_workspace_size(B, H, N, d)
        rows = B * H * ((N + 127) // 128 * 128)
        expect = (2 * rows * 4 + 255) // 256 * 256 + 256 + (B * H * N * tile * 4 + 255) // 256 * 256
        assert ws == expect
        assert lib.fa2_bwd_ex_workspace_size(B, H, N, d, 1) == (2 * rows * 4 + 255) // 256 * 256 + 256
        # O(B H N d): at most 8 bytes per head element plus the row statistics
        assert ws <= B * H * N * (8 * d) + 2 * rows * 4 + 768
        # all but the counter doubles with N
        assert lib.fa2_bwd_workspace_size(B, H, 2 * N, d) - 256 == 2 * (ws - 256)


def test_noalloc_rejects_sizes_beyond_its_buffer_before_any_device_call(lib):
    # the training shape (8 x 16 heads of 4096 rows, d = 128) needs 258 MiB of scratch
    B, H, N, d = 8, 16, 4096, 128
    assert lib.fa2_bwd_workspace_size(B, H, N, d) > (32 << 20) - 256
    far = 1 << 33  # fake pointers 8 GiB apart: the tensors do not overlap
    ptrs = [far * (i + 1) for i in range(9)]
    assert lib.fa2_bwd_noalloc(*ptrs, B, H, N, d, 0.1, 0, 1, None) == fa2.FA2_ERR_WORKSPACE


def test_bwd_ex_validation_without_device(lib):
    ptrs = [P * (i + 1) for i in range(9)]
    ws = fa2.fa2_bwd_ex_workspace_size(1, 1, 64, 64, fa2.FA2_BWD_DETERMINISTIC)
    # unknown flag, negative window, a window without causal
    assert lib.fa2_bwd_ex(*ptrs, 16 * P, ws, 1, 1, 64, 64, 0.1, 1, 0, 2, 1, None) == fa2.FA2_ERR_INVALID_ARG
    assert lib.fa2_bwd_ex(*ptrs, 16 * P, ws, 1, 1, 64, 64, 0.1, 1, -1, 1, 1, None) == fa2.FA2_ERR_INVALID_ARG
    assert lib.fa2_bwd_ex(*ptrs, 16 * P, ws, 1, 1, 64, 64, 0.1, 0, 8, 1, 1, None) == fa2.FA2_ERR_INVALID_ARG
    # the deterministic mode's workspace is the smaller one; too small is still rejected
    assert lib.fa2_bwd_ex(*ptrs, 16 * P, ws - 256, 1, 1, 64, 64, 0.1, 1, 0, 1, 1, None) == fa2.FA2_ERR_WORKSPACE
    # head dims end at 128 in both modes
    assert lib.fa2_bwd_ex(*ptrs, 16 * P, 1 << 20, 1, 1, 64, 136, 0.1, 1, 0, 1, 1, None) == fa2.FA2_ERR_UNSUPPORTED
