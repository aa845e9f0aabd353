"""Host-side accounting of the benchmark, on CPU: the kept-block FLOP count,
the clock-record summary and the staleness rule of the stored DRAM counters."""
import json
import os

import numpy as np
import pytest
import torch

import bench


def _brute_force_kept_flops(kv_idx, kv_cnt, N, d, bq, bk):
    """4*d times the number of (query token, key token) pairs the mask keeps,
    counted token by token."""
    B, H, nqb, _ = kv_idx.shape
    total = 0
    for b in range(B):
        for h in range(H):
            keep = np.zeros((N, N), bool)
            for I in range(nqb):
                for J in kv_idx[b, h, I, : kv_cnt[b, h, I]]:
                    keep[I * bq:(I + 1) * bq, J * bk:(J + 1) * bk] = True
            total += int(keep.sum())
    return 4.0 * d * total


@pytest.mark.parametrize("N,bq,bk", [(200, 64, 32), (256, 128, 64), (130, 64, 128), (64, 64, 64)])
def test_kept_flops_counts_valid_token_pairs(N, bq, bk):
    rng = np.random.default_rng(N + bq + bk)
    B, H, d = 2, 3, 64
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx = np.full((B, H, nqb, nkb), -7, np.int32)  # entries past the count are never read
    kv_cnt = rng.integers(0, nkb + 1, size=(B, H, nqb)).astype(np.int32)
    for b in range(B):
        for h in range(H):
            for I in range(nqb):
                c = kv_cnt[b, h, I]
                kv_idx[b, h, I, :c] = np.sort(rng.choice(nkb, size=c, replace=False))
    got = bench.kept_flops(torch.from_numpy(kv_idx), torch.from_numpy(kv_cnt), N, d, bq, bk)
    assert got == _brute_force_kept_flops(kv_idx, kv_cnt, N, d, bq, bk)


def test_kept_flops_all_blocks_is_dense():
    N, d, bq, bk = 300, 128, 128, 64
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx = torch.arange(nkb, dtype=torch.int32).repeat(1, 2, nqb, 1)
    kv_cnt = torch.full((1, 2, nqb), nkb, dtype=torch.int32)
    assert bench.kept_flops(kv_idx, kv_cnt, N, d, bq, bk) == 4.0 * 2 * N * N * d


def test_clock_summary_median_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 1000.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    c.lines = ["0, 1000, 1965, 500, 0x8, Active, Not Active, Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    c.lines = []
    assert c.summary()["sm_mhz"] is None


def test_stored_traffic_is_dropped_once_the_kernel_changes(tmp_path, monkeypatch):
    csrc = tmp_path / "block_sparse_attention_pooled_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "attn.cuh").write_text("// kernel v1\n")
    (csrc / "ptx.cuh").write_text("// helpers\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    kernel = "attn_fwd_kernel<128, 0>"
    entry = {"dram_bytes_per_launch": 123.0, "kernel": kernel, "csrc_sha": bench.kernel_source_sha(kernel)}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"480p": entry}))
    assert bench.dram_traffic("480p", kernel) == 123.0
    assert bench.dram_traffic("720p", kernel) is None  # no capture for this workload
    assert bench.dram_traffic("480p", "attn_fwd_kernel<128, 1>") is None  # another kernel
    (csrc / "attn.cuh").write_text("// kernel v2\n")
    assert bench.dram_traffic("480p", kernel) is None


def test_peaks_fall_back_when_no_measurement(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.measured_peaks()
    assert kind == "fallback" and peaks["bf16_tflops"] > peaks["bf16_tflops_sustained"] > 0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1.0, "hbm_gbs": 2.0}))
    peaks, kind = bench.measured_peaks()
    assert kind == "measured" and peaks["bf16_tflops"] == 1.0


def test_committed_traffic_entries_name_their_capture():
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as f:
        entries = json.load(f)
    for name, e in entries.items():
        assert e["dram_bytes_per_launch"] > 0 and e["kernel"].split("<")[0] in bench.KERNEL_SOURCES, name
        assert os.path.exists(os.path.join(bench.ROOT, e["source"])), name


def test_burst_peak_applies_at_max_clock_or_without_samples(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
                                                              "hbm_gbs": 6000.0}))
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "samples": 9}
    capped = {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "samples": 9}
    none = {"sm_mhz": None, "sm_max_mhz": None, "samples": 0}
    assert bench.clocks_at_max(at_max) and bench.clocks_at_max(none) and not bench.clocks_at_max(capped)
    peak, fr, desc = bench.roofline_peak(800.0, at_max)
    assert peak == 1600.0 and "burst" in desc and fr["frac_vs_burst"] == 0.5 and fr["frac_vs_sustained"] == 800 / 1400
    assert fr["frac_vs_nominal"] == 800.0 / bench.NOMINAL_BF16_TFLOPS
    peak, _, desc = bench.roofline_peak(800.0, none)
    assert peak == 1600.0 and "no clock samples" in desc
    peak, _, desc = bench.roofline_peak(800.0, capped)
    assert peak == 1400.0 and "sustained" in desc
    peak, fr, _ = bench.roofline_peak(800.0, at_max, ratio=2.0)
    assert peak == 3200.0 and fr["frac_vs_burst"] == 0.25


def test_timed_steps_flush_outside_each_steps_events():
    """Every step is preceded by an L2 flush that lies outside its own events,
    and each step records its span events between them."""
    log = []

    class Ev:
        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            self.t = len(log)
            log.append("ev")

        def elapsed_time(self, other):
            return float(other.t - self.t)

    class Flush:
        def zero_(self):
            log.append("flush")

    class Cuda:
        Event = Ev

        @staticmethod
        def synchronize():
            log.append("sync")

    def step(ea, eb):
        ea.record()
        log.append("work")
        eb.record()

    step_ms, attn_ms = bench.timed_steps(step, 3, None, Flush(), cuda=Cuda)
    assert log == ["flush", "ev", "ev", "work", "ev", "ev"] * 3 + ["sync"]
    assert step_ms == [4.0] * 3 and attn_ms == [2.0] * 3


def test_nvml_sampler_falls_back_without_a_gpu():
    with bench.NvmlClockSampler("GPU-00000000-0000-0000-0000-000000000000", period_s=0.001) as clk:
        pass
    s = clk.summary()
    assert "samples" in s and "source" in s
