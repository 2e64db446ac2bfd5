"""Device memory of the calls: nothing allocated per call, scratch linear in N.

"FlashAttention-2" (systems-analysis.info wiki), "Предпосылки": the tiled method
needs memory linear in the sequence length, since no N x N matrix is stored.  Here
the caller owns every tensor and the backward's workspace; the library itself
allocates one status word per device on its first call and nothing after that.
Free device memory is read with cudaMemGetInfo around each call (every tensor is
allocated before the first reading, and every kernel has run once, so lazy module
loading does not count).
"""

import math

import pytest
import torch

from exact_io_aware_74_b200 import fa2
from exact_io_aware_74_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_calls_allocate_nothing_and_workspace_is_linear(d):
    B, H = 1, 4
    scale = 1 / math.sqrt(d)
    ws_sizes = {}
    for N in (1024, 2048, 4096, 8192):
        x = make_inputs(B, H, N, d, "bf16", seed=50 + N, with_do=True)
        q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
        o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        ws_sizes[N] = fa2.fa2_bwd_workspace_size(B, H, N, d)
        ws = torch.empty(ws_sizes[N], dtype=torch.uint8, device="cuda")

        def step():
            assert fa2.fa2_fwd(q, k, v, o, lse, scale, True) == fa2.FA2_OK
            assert fa2.fa2_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, scale, True) == fa2.FA2_OK
            assert fa2.fa2_get_device_status() == (fa2.FA2_OK, 0)

        step()  # first launch of these kernels (lazy loading) and of the status word
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0, f"N={N}: device memory changed"
        del q, k, v, do, o, dq, dk, dv, lse, ws
    # the only N-dependent memory besides the caller's tensors: linear, not quadratic
    # (all of it but the 256-byte tile counter scales with N)
    assert ws_sizes[2048] - 256 == 2 * (ws_sizes[1024] - 256)
    assert ws_sizes[8192] - 256 == 8 * (ws_sizes[1024] - 256)
    assert ws_sizes[8192] < 8192 * 8192  # far below one N x N byte matrix per head
