"""Host-side pieces of bench.py that decide what the JSON line says, on CPU:
the clock record of the timed region, the recorded DRAM traffic and when it
stops applying, the measured-peak file and its fallback, the causal pair
count behind the FLOP figures, and the reference (CPU oracle) arm's line."""
import json
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


class _Thread:
    def join(self, timeout=None):
        pass


def _record(lines, window):
    s = bench.ClockSampler(0)
    s.proc, s.thread = _Proc(), _Thread()
    s.lines = lines
    s.stop()
    return s.summary(*window)


def _line(sm, cap="Not Active", hw="Not Active", mask="0x0000000000000000"):
    return f"{sm}, 1965, 900.5, {cap}, {hw}, Not Active, Not Active, {mask}"


def test_clock_record_keeps_only_the_timed_window(monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    lines = [(0.5, _line(1965)),                                     # before the window: idle clocks
             (1.0, _line(1600, cap="Active", mask="0x0000000000000004")),
             (1.5, _line(1620, cap="Active", mask="0x0000000000000004")),
             (2.0, _line(1610)),
             (2.05, "garbled"),                                        # malformed: skipped
             (3.0, _line(700, hw="Active", mask="0x0000000000000008"))]  # after the window
    rec = _record(lines, (1.0, 2.0))
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1610.0 and rec["sm_max_mhz"] == 1965.0
    assert (rec["sm_mhz_min"], rec["sm_mhz_max"]) == (1600.0, 1620.0)
    assert rec["reasons"] == ["sw_power_cap"]                        # hw_slowdown came after the window
    assert rec["active_masks"] == ["0x0", "0x4"]


def test_clock_records_of_two_windows(monkeypatch):
    """One sampler serves several timed windows (the headline and each other workload)."""
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    lines = [(1.0, _line(1900)), (1.5, _line(1880)), (3.0, _line(1500, cap="Active", mask="0x0000000000000004"))]
    s = bench.ClockSampler(0)
    s.proc, s.thread = _Proc(), _Thread()
    s.lines = lines
    a, b = s.summary(0.9, 1.6), s.summary(2.9, 3.1)
    assert (a["samples"], a["sm_mhz"], a["reasons"]) == (2, 1890.0, [])
    assert (b["samples"], b["sm_mhz"], b["reasons"]) == (1, 1500.0, ["sw_power_cap"])


def test_clock_peak_is_the_tensor_rate_at_the_sampled_clock():
    assert bench.clock_peak_tflops(None) is None
    # 8192 flop per clock per SM x 148 SMs at 1.85 GHz: the nominal 2.24 PFLOP/s dense bf16
    assert bench.clock_peak_tflops(1850.0) == pytest.approx(8192 * 148 * 1.85e9 / 1e12)


def test_clock_record_names_reasons_from_the_mask(monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    lines = [(1.0, _line(1200, mask="0x0000000000000048"))]           # hw_slowdown | hw_thermal_slowdown
    rec = _record(lines, (0.0, 5.0))
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_clock_record_without_nvidia_smi():
    s = bench.ClockSampler(0)
    s.stop()
    rec = s.summary(0.0, 1.0)
    assert rec["sm_mhz"] is None and rec["reasons"] == ["nvidia-smi unavailable"]


def test_recorded_traffic_applies_only_to_its_workload_and_sources(monkeypatch):
    rec = {"workload": "roundtrip_p4_n128k", "bytes_per_launch": 123456789,
           "sources_sha256": bench.sources_sha256("attn_bwd_dkdv_kernel")}
    monkeypatch.setitem(bench.TRAFFIC, "attn_bwd_dkdv_kernel", rec)
    assert bench.recorded_traffic("attn_bwd_dkdv_kernel", rec["workload"]) == rec["bytes_per_launch"]
    assert bench.recorded_traffic("attn_bwd_dkdv_kernel", "llama8b_p4_n32k") is None
    monkeypatch.delitem(bench.TRAFFIC, "attn_bwd_dq_kernel", raising=False)
    assert bench.recorded_traffic("attn_bwd_dq_kernel", rec["workload"]) is None   # no record
    # once the kernel's sources differ from the ones the counters were taken on
    monkeypatch.setitem(bench.TRAFFIC, "attn_bwd_dkdv_kernel", dict(rec, sources_sha256="0" * 64))
    assert bench.recorded_traffic("attn_bwd_dkdv_kernel", rec["workload"]) is None


def test_every_recorded_traffic_matches_the_current_sources():
    """A committed record whose kernel has changed since the capture would be
    reported as null: keep only records of the current sources."""
    for kernel, rec in bench.TRAFFIC.items():
        assert rec["sources_sha256"] == bench.sources_sha256(kernel), kernel


def test_sources_hash_covers_the_kernel_region(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("head\nnamespace dkdv {\nbody\n}  // namespace dkdv\ntail\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "k", (("k.cu", "namespace dkdv {", "}  // namespace dkdv"),))
    h0 = bench.sources_sha256("k")
    src.write_text("other head\nnamespace dkdv {\nbody\n}  // namespace dkdv\nother tail\n")
    assert bench.sources_sha256("k") == h0                           # outside the region: same kernel
    src.write_text("head\nnamespace dkdv {\nbody2\n}  // namespace dkdv\ntail\n")
    assert bench.sources_sha256("k") != h0


def test_peaks_from_file_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks()["source"] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6500, "bf16_tflops": 1600}))
    pk = bench.load_peaks()
    assert pk == {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1600.0, "source": "measured"}


@pytest.mark.parametrize("lengths", [[[1]], [[5, 3]], [[128, 1, 7], [100]]])
def test_pair_count_is_the_causal_segmented_mask(lengths):
    """pairs = number of (query, key) pairs with key <= query in the same sample."""
    brute = 0
    for row in lengths:
        seg = [i for i, L in enumerate(row) for _ in range(L)]
        brute += sum(1 for i in range(len(seg)) for j in range(i + 1) if seg[i] == seg[j])
    assert bench.pairs_of(lengths) == brute


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the CPU oracle arm) prints one JSON line
    with the keys the driver reads, on a small workload."""
    import os
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_p2_n256", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, env=dict(os.environ, RANK="0"))
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["unit"] == "TFLOP/s" and out["value"] > 0
    assert out["metric"] == bench.METRIC and out["higher_is_better"] is True
    assert (out["steps"], out["warmup"], out["n_gpus"]) == (2, 1, 1)
    assert out["config"]["workload"] == "tiny_p2_n256"
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"] == {"value": out["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
