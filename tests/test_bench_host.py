"""Host logic of bench.py on CPU: FLOP accounting, peaks, the max-over-ranks
aggregation (two gloo ranks), the reference arm and the traffic record lookup."""

import json
import os
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from exact_io_aware_74_b200.workloads import WORKLOADS  # noqa: E402


def test_step_flops_and_default_workload():
    w = WORKLOADS[bench.DEFAULT_WORKLOAD]
    # the largest forward + backward workload: B=8, H=16, N=4096, d=128, causal
    assert w.backward and w.dtype == "bf16" and w.causal
    assert (w.B, w.H, w.N, w.d) == (8, 16, 4096, 128)
    assert bench.step_flops(w) == pytest.approx(3.5 * 4 * 8 * 16 * 4096 * 4096 * 128 / 2)
    # its inputs are larger than L2, so no flush buffer is written between steps
    assert bench.input_bytes(w) * 2 >= 2 * bench.L2_BYTES
    assert bench.HEADLINE_WORKLOAD == "fwd_bf16_b2h32_n8192_d128"


def test_load_peaks_measured_and_fallback(tmp_path):
    p = tmp_path / "peaks.json"
    p.write_text(json.dumps({"hbm_gbs": 6000, "bf16_tflops": 1600, "bf16_tflops_sustained": 1400}))
    peaks, src = bench.load_peaks(str(p))
    assert src == "measured" and peaks["bf16_tflops"] == 1600
    peaks, src = bench.load_peaks(str(tmp_path / "missing.json"))
    assert src == "fallback" and peaks["bf16_tflops"] == 1590.0


def _agg_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    t, f = bench.aggregate(1.0 + rank, 10.0 * (rank + 1), world)
    q.put((rank, t, f))
    torch.distributed.destroy_process_group()


def test_aggregate_takes_max_time_and_total_flops_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_agg_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=60) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, t, f in res:
        assert t == 2.0 and f == 30.0


def test_aggregate_is_identity_without_process_group():
    assert bench.aggregate(3.0, 7.0, 1) == (3.0, 7.0)


def test_traffic_record_requires_current_kernel_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (tmp_path / "exact_io_aware_74_b200").mkdir()
    csrc = tmp_path / "exact_io_aware_74_b200" / "csrc"
    csrc.mkdir()
    for name in sorted({n for srcs in bench.KERNEL_SOURCES.values() for n in srcs}):
        (csrc / name).write_text(name + " v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.csrc_hash("fa2_bwd")
    (prof / "dram_traffic.txt").write_text(f"fa2_bwd:w {h} 12345\nfa2_fwd:w deadbeef 99\n")
    assert bench.traffic_from_profiles("fa2_bwd:w") == 12345
    assert bench.traffic_from_profiles("fa2_fwd:w") is None
    (csrc / "fa2_fwd.cuh").write_text("fa2_fwd.cuh v2")   # another kernel: record stands
    assert bench.traffic_from_profiles("fa2_bwd:w") == 12345
    (csrc / "fa2_bwd.cuh").write_text("fa2_bwd.cuh v2")   # this kernel changed: void
    assert bench.traffic_from_profiles("fa2_bwd:w") is None


def test_clock_sampler_summary_decodes_reasons():
    s = bench.ClockSampler(0)
    s.samples = [(1900, 0x4), (1800, 0x0), (1850, 0x1)]
    s.max_mhz = 1965
    out = s.summary()
    assert out["sm_mhz"] == 1850 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]


def test_reference_arm_prints_one_json_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "fwd_fp16_b1h2_n128_d64", "--steps", "2", "--warmup", "0"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["value"] > 0 and out["unit"] == "TFLOP/s"
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["e2e"]["h2d_bytes_per_step"] == 0
