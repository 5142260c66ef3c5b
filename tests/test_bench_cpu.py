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
    (tmp_path / "profiles" / "c.md").write_text(
        f"# z\n\nkernel: score_stream\nworkload: w4\nsource_sha: {sha}\n"
        "dram_bytes_per_query: 93800\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "score_src_sha", lambda kernel="score_stream": sha)
    assert bench.profile_traffic("score_stream", "w1") == ("pair", 1.5)
    assert bench.profile_traffic("score_stream", "w2") is None     # stale hash
    assert bench.profile_traffic("score", "w1") is None            # other kernel
    assert bench.profile_traffic("score_stream", "w3") is None     # no summary
    assert bench.profile_traffic("score_stream", "w4") == ("query", 93800.0)


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


def test_recall_and_iou_rows_match_the_oracle_definition():
    import numpy as np
    import torch

    import oracle
    A = np.array([[1, 2, 3, -1], [5, 6, 7, 8], [-1, -1, -1, -1], [4, 9, -1, -1]], np.int32)
    D = np.array([[3, 2, 9, -1], [8, 7, 6, 5], [-1, -1, -1, -1], [1, 2, 3, 0]], np.int32)
    rec, iou = bench.recall_iou_rows(torch.from_numpy(A), torch.from_numpy(D))
    # row 2 is skipped (empty dense selection)
    want = [oracle.recall_iou(A[i], D[i]) for i in (0, 1, 3)]
    assert abs(rec - np.mean([r for r, _ in want])) < 1e-12
    assert abs(iou - np.mean([u for _, u in want])) < 1e-12
    # random rows of distinct indices with padding
    rng = np.random.default_rng(0)
    rows_a, rows_d = [], []
    for _ in range(50):
        n = int(rng.integers(1, 40))
        a = rng.choice(60, size=n, replace=False)
        d = rng.choice(60, size=int(rng.integers(1, 40)), replace=False)
        rows_a.append(np.pad(a, (0, 40 - len(a)), constant_values=-1))
        rows_d.append(np.pad(d, (0, 40 - len(d)), constant_values=-1))
    A, D = np.array(rows_a, np.int32), np.array(rows_d, np.int32)
    rec, iou = bench.recall_iou_rows(torch.from_numpy(A), torch.from_numpy(D))
    want = [oracle.recall_iou(A[i], D[i]) for i in range(len(A))]
    assert abs(rec - np.mean([r for r, _ in want])) < 1e-12
    assert abs(iou - np.mean([u for _, u in want])) < 1e-12


def test_split_prof_separates_counters_from_kernels():
    kern, cnt = bench.split_prof({"score": (1.5, 2), "#rescan_queries": (0.0, 7),
                                  "select": (0.5, 1)})
    assert kern == {"score": (1.5, 2), "select": (0.5, 1)}
    assert cnt == {"rescan_queries": 7}


def test_roofline_uses_the_burst_peak_for_prefill_and_hbm_for_decode():
    from misa_synth import make_workload
    wl = make_workload(seq_lens=[4096], queries="all", H=8, B=64, m=8, k=16, seed=1)
    peaks = {"bf16": 1600.0, "bf16_sustained": 1400.0, "hbm_gbs": 6500.0, "source": "test"}
    r = bench.roofline_of(wl, 2.0, 1, True, peaks, {"sm_mhz": 1800.0}, "none")
    flops = 2 * 8 * 128 * wl.pairs
    assert abs(r["achieved"] - flops / 2e-3 / 1e12) < 1e-9
    assert r["peak"] == 1600.0 and abs(r["frac"] - r["achieved"] / 1600.0) < 1e-12
    assert abs(r["frac_of_sustained"] - r["achieved"] / 1400.0) < 1e-12
    wl2 = make_workload(seq_lens=[1000, 500], queries=3, H=8, B=64, m=8, k=16, seed=1)
    r2 = bench.roofline_of(wl2, 0.01, 1, False, peaks, {}, "none")
    abytes = (1000 + 500) * 256 + 4 * wl2.pairs
    assert r2["bound"] == "hbm" and abs(r2["achieved"] - abytes / 1e-5 / 1e9) < 1e-6


def test_streamed_rule_follows_the_selection_pass():
    # prefill (streaming pass + selection), decode (score rows + row top-k) and
    # the MISA-dagger prefill (streamed keep, then the re-rank's row top-k)
    assert bench.is_streamed({"route": 1, "score": 1, "select": 1})
    assert not bench.is_streamed({"route": 1, "score": 1, "topk": 1})
    assert bench.is_streamed({"score": 1, "select": 1, "rerank_score": 1, "topk": 1})
