"""Host logic of bench.py: rank reduction over gloo (world size 2), roofline figures,
and the oracle arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as W  # noqa: E402


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w = bench.dist_setup("gloo")
    bench.barrier()
    got = bench.max_over_ranks(1.5 + r)
    rate = bench.whole_job_rate(100.0, w, got)
    out.put((r, w, got, rate))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[2] for r in res] == [2.5, 2.5]          # the slowest rank's time on both
    assert [r[3] for r in res] == [80.0, 80.0]        # 2 ranks x 100 units / 2.5 s


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_rate(10.0, 1, 2.0) == 5.0


def test_algorithmic_figures_of_7b_shapes():
    wl = W.WORKLOADS[W.HEADLINE]
    flops, bytes_, upd = bench.algorithmic(wl)
    assert wl.params == 6_476_005_376
    assert abs(flops / 1.35e13 - 1) < 0.01
    assert abs(bytes_ / 219.1e9 - 1) < 0.01
    assert upd == 20 * wl.params


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "single_256x128_r32", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "params/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    # one matrix is the whole workload here: nothing extrapolated
    assert d["extrapolated"] is False and d["matrices_run_per_step"] == 1


def test_reference_arm_marks_extrapolation():
    """On a multi-matrix workload the oracle arm runs one matrix per bucket, scales it by
    the bucket counts, and says so in fields of its own."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "fullrank_16x1024x1024", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][0])
    assert d["extrapolated"] is True
    assert d["matrices_run_per_step"] == 1 and d["matrices_per_workload_step"] == 16
    assert d["sample_ms_per_step"] < d["ms_per_step"]


def test_clock_summary_flags_throttle_reasons():
    """Samples (MHz, max MHz, W, reason bits): the median is taken over loaded samples
    (power above 200 W) and every throttle reason seen is named."""
    rows = [(1965, 1965, 150.0, 0), (1800, 1965, 900.0, 0x4), (1700, 1965, 950.0, 0x4),
            (1900, 1965, 800.0, 0x40)]
    s = bench.summarize_clocks(rows, "test")
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["samples"] == 4
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert bench.summarize_clocks([])["reasons"] == ["clocks not sampled"]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "single_256x128_r32", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_split_ceiling_of_the_rank_sweep():
    """fp32 mode's ceiling counts the bf16 products its splits issue (36 m n r + 18 m r^2)
    and 40 B per weight element; at r = 1024 on 8 x 8192^2 the products dominate."""
    wl = W.WORKLOADS["square_8x8192_r1024"]
    peaks = {"bf16_tflops": 1672.0, "hbm_gbs": 6458.1}
    f, b, t = bench.split_ceiling(wl, peaks)
    m = n = 8192
    r = 1024
    assert f == 8 * (36 * m * n * r + 18 * m * r * r + r ** 3 / 3)
    assert b == 8 * (40 * m * n + 4 * (3 * m * r + 6 * n * r))
    assert t == f / 1672e12 and f / 1672e12 > b / 6458.1e9


def test_update_traffic_comes_from_captures_of_this_kernel():
    """The per-shape DRAM figures behind `roofline.traffic` were captured on the update
    kernel as committed (its source hash), each figure is read + write over elements of
    its capture, and the 7B-like step's traffic per launch is their element-weighted
    mean over the three launches."""
    per, h = bench.update_traffic()
    assert per is not None and h == bench.update_kernel_hash()
    caps = json.load(open(bench.TRAFFIC_FILE))["captures"]
    for shape, c in caps.items():
        assert abs(per[shape] - (c["dram_read"] + c["dram_write"]) / c["elements"]) < 1e-9
    wl = W.WORKLOADS[W.HEADLINE]
    want = sum(per[f"{b.m}x{b.n}"] * b.params for b in wl.buckets) / len(wl.buckets)
    assert bench.update_traffic_per_launch(wl, len(wl.buckets)) == pytest.approx(want)
    assert 20.0 * wl.params / 3 <= want <= 21.0 * wl.params / 3


def test_update_traffic_is_null_once_the_kernel_changes(monkeypatch):
    wl = W.WORKLOADS[W.HEADLINE]
    monkeypatch.setattr(bench, "update_kernel_hash", lambda: "0" * 16)
    assert bench.update_traffic_per_launch(wl, 3) is None
