"""Host logic of bench.py: the roofline's algorithmic bytes counted by hand on tiny cases, the
profile-traffic match, the clock summary of nvidia-smi rows, and the HBM peak's source."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_by_hand():
    # one sequence of 40 tokens (3 pages), 4 q-heads / 2 kv-heads
    seq_lens = np.array([40])
    sel = np.full((1, 4, 2), -1)
    cnt = np.array([[1, 2, 2, 1]])
    sel[0, 0, :1] = [0]
    sel[0, 1, :2] = [0, 2]          # group 0 union of pages: {0, 2}
    sel[0, 2, :2] = [1, 2]
    sel[0, 3, :1] = [1]             # group 1 union: {1, 2}
    union_count = np.array([[5, 7]])
    total, parts = bench.algorithmic_bytes(None, seq_lens, 4, 2, sel, cnt, union_count)
    assert parts["bounds"] == 3 * 2 * 512
    assert parts["page_table"] == 3 * 4
    assert parts["int4"] == (2 + 2) * 1088
    assert parts["kv"] == (5 + 7) * 512
    assert parts["q_o"] == 4 * (256 + 516) + 4
    assert total == sum(parts.values())


def test_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    assert bench.measured_traffic() in (None,) or isinstance(bench.measured_traffic(), int)
    monkeypatch.setattr(bench, "source_hash", lambda kernel="decode_step": "not-the-sources")
    assert bench.measured_traffic() is None
    assert bench.measured_traffic("prune_rows", "dram_bytes_per_launch_n131072") is None


def test_prune_rows_bytes_by_hand():
    # 3 rows of 8 weights: 4 B per weight read, m and the count written (8 B per row), 4 B per
    # kept index when the indices are written
    assert bench.prune_rows_bytes(8, 3, 5, False) == 3 * (32 + 8)
    assert bench.prune_rows_bytes(8, 3, 5, True) == 3 * (32 + 8) + 20


def test_clock_summary_from_nvidia_smi_rows():
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1905, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 10.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # skipped
        "garbage",
    ]
    out = bench.ClockSampler.summarise(rows)
    assert out == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}
    hot = rows[:1] + ["0, 1200, 1965, 800, 0x8, Active, Not Active, Active, Not Active"]
    assert bench.ClockSampler.summarise(hot)["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler.summarise([])["sm_mhz"] is None


def test_hbm_peak_measured_or_fallback(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6554.9, "bf16_tflops": 1500}')
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.hbm_peak() == (6554.9, "measured")
    (tmp_path / "MEASURED_PEAKS.json").unlink()
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")


def test_host_info_reads_the_model_name(tmp_path):
    f = tmp_path / "cpuinfo"
    f.write_text("processor\t: 0\nvendor_id\t: X\nmodel name\t: Some CPU @ 2.0GHz\nflags\t: a\n")
    info = bench.host_info(str(f))
    assert info["model"] == "Some CPU @ 2.0GHz" and info["nproc"] == os.cpu_count()
    assert bench.host_info(str(tmp_path / "missing"))["model"] is None


def test_configs_name_their_workload_and_l2_policy():
    for name in bench.WORKLOADS:
        cfg = bench.workload_config(name)
        assert cfg["workload"] and "l2" in cfg and "model" not in cfg
    cfg = bench.prune_rows_config([8192, 131072], {8192: 4, 131072: 1})
    assert cfg["rows"] == 4096 and cfg["n"] == [8192, 131072] and "l2" in cfg
    assert bench.append_config()["workload"]


def test_bench_help_runs_without_a_gpu():
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "--workload" in r.stdout and "--impl" in r.stdout
