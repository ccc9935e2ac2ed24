"""Host-side contract of bench.py's JSON lines (CPU only).

The reference arm (`bench.py --impl reference`) times the CPU oracle on a
bounded sample of the decode workload and prints one JSON line on rank 0.
This checks the keys the line must carry and that its numbers agree with
each other, on the smallest sample the arm takes.
"""
import contextlib
import io
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    return bench


def test_reference_arm_prints_one_complete_line():
    bench = _bench()
    args = type("A", (), dict(warmup=0, steps=1, ref_seconds=0.0, gpus=1))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, 1, 0)
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["config"]["workload"] == bench.WORKLOAD
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["n_gpus"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["unit"] == "GB/s"
    assert int(cb["cores"]) >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_job_throughput_is_bytes_over_the_slowest_rank():
    bench = _bench()
    # 4.34 MB per launch x 120 launches per step, 200 steps, one rank, 76 ms
    step_bytes = 4341760 * 120
    v = bench.job_throughput(step_bytes, 200, 1, 0.076)
    assert abs(v - step_bytes * 200 / 0.076 / 1e9) < 1e-9
    # two ranks: twice the bytes over the same (max) time
    assert abs(bench.job_throughput(step_bytes, 200, 2, 0.076) - 2 * v) < 1e-9


def test_clock_summary_reads_median_clock_and_active_reasons():
    bench = _bench()
    cs = bench.ClockSampler(0)          # no GPU here: only the parser is used
    cs.out.write("0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n")
    cs.out.write("0, 1320, 1965, 999.8, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n")
    cs.out.write("0, 1950, 1965, 880.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n")
    cs.out.write("garbage line\n")
    s = cs.summary()
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_samples_says_so():
    bench = _bench()
    cs = bench.ClockSampler(0)
    s = cs.summary()
    assert s["sm_mhz"] is None and s["reasons"] == ["unavailable"]


def test_cpu_baseline_reports_all_cores_one_core_and_prefill():
    """The CPU baseline of the GPU arm: the best of three all-core samples,
    one single-core sample and a prefill timing, each with its own cores."""
    bench = _bench()
    import oracle
    cores = oracle.num_threads()
    cb = bench.cpu_baseline(0.0)
    assert cb["kind"] == "oracle" and cb["unit"] == "GB/s"
    assert len(cb["runs_GBps"]) == 3 and cb["value"] == max(cb["runs_GBps"])
    assert int(cb["cores"]) == cores
    assert cb["one_core"]["cores"] == 1 and cb["one_core"]["value"] > 0
    assert cb["prefill"]["TOPS"] > 0 and cb["prefill"]["M"] == 64
    assert oracle.num_threads() == cores          # the thread count is restored


def test_gemv_path_names_every_kernel():
    """bench.py's path names cover every kernel the library's plan can report."""
    bench = _bench()
    import bit_ternary_weight_b200 as bl
    src = open(os.path.join(ROOT, "bench.py")).read()
    for kern in bl.GEMV_KERNELS.values():
        assert f'"{kern}":' in src, kern
