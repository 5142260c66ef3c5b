"""Host-side measurement logic of bench.py on CPU (no GPU): clock-sample
summaries, the profile-traffic lookup by kernel source hash, and the CPU
baseline's sampling of the oracle."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _clocks(lines, i0, i1):
    c = bench.Clocks("GPU-test")
    c.proc = None
    c.lines = lines
    c.i0, c.i1 = i0, i1
    return c


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


class _DoneThread:
    def join(self, timeout=None):
        pass


def test_clock_summary_counts_only_samples_inside_the_region():
    row = "{sm}, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, {cap}"
    lines = [row.format(sm=600, cap="Not Active"),          # before the region
             row.format(sm=1800, cap="Active"),
             row.format(sm=1900, cap="Not Active"),
             row.format(sm=1700, cap="Active"),
             row.format(sm=500, cap="Not Active")]          # after the region
    c = _clocks(lines, 1, 4)
    c.proc, c.t = _DoneProc(), _DoneThread()
    out = c.stop()
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1800.0          # median of 1800, 1900, 1700
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert "note" not in out


def test_clock_summary_of_a_short_region_takes_the_next_sample():
    row = "1850, 1965, 950.0, 0x0, Not Active, Active, Not Active, Not Active"
    c = _clocks([row, row], 1, 1)            # no sample fell inside the region
    c.proc, c.t = _DoneProc(), _DoneThread()
    out = c.stop()
    assert out["samples"] == 1
    assert out["reasons"] == ["hw_thermal_slowdown"]
    assert "sampling period" in out["note"]


def test_profile_traffic_lookup_matches_kernel_workload_and_source_hash(tmp_path, monkeypatch):
    sha = bench.score_src_sha("score_stream")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "a.md").write_text(
        f"# x\n\nkernel: score_stream\nworkload: w1\nsource_sha: {sha}\n"
        "dram_bytes_per_pair: 1.5\n")
    (tmp_path / "profiles" / "b.md").write_text(
        "# y\n\nkernel: score_stream\nworkload: w2\nsource_sha: 0000000000000000\n"
        "dram_bytes_per_pair: 9.0\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "score_src_sha", lambda kernel="score_stream": sha)
    assert bench.traffic_per_pair("score_stream", "w1") == 1.5
    assert bench.traffic_per_pair("score_stream", "w2") is None     # stale hash
    assert bench.traffic_per_pair("score", "w1") is None            # other kernel
    assert bench.traffic_per_pair("score_stream", "w3") is None     # no summary


def test_source_hash_depends_on_the_kernel():
    a, b = bench.score_src_sha("score_stream"), bench.score_src_sha("score")
    assert len(a) == 16 and len(b) == 16 and a != b


def test_cpu_baseline_samples_the_oracle_on_all_cores_and_one_thread():
    from misa_synth import make_config
    wl = make_config(0)
    out = bench.cpu_oracle_sample(wl, 0.2, one_core_s=0.1)
    assert out["kind"] == "oracle" and out["unit"] == bench.UNIT
    assert out["value"] > 0 and out["cores"] >= 1
    assert "value_1core" in out and out["value_1core"] > 0
    assert out["cpu_model"]


def test_mean_recall_of_two_selections():
    import numpy as np
    A = np.array([[1, 2, 3, -1], [5, 6, 7, 8], [-1, -1, -1, -1]])
    D = np.array([[3, 2, 9, -1], [8, 7, 6, 5], [-1, -1, -1, -1]])
    # row 0: {2,3} of {2,3,9}; row 1: all four; row 2 skipped (empty D)
    assert abs(bench.mean_recall(A, D) - (2 / 3 + 1.0) / 2) < 1e-12
    assert bench.mean_recall(D[2:], D[2:]) == 1.0
