"""Host-side arithmetic of bench.py (CPU): the work per step, the per-kernel
breakdown and the peaks it divides by.  No GPU is involved."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_step_flops_closed_form():
    # 28 layers x 4 linears x 3 GEMMs (fprop, dgrad, wgrad), 2 T n k each
    T = 8192
    per_layer = sum(3 * 2 * T * n * k for n, k in ((4096, 2048), (2048, 2048), (12288, 2048), (2048, 6144)))
    assert bench.step_gemm_flops(28) == pytest.approx(28 * per_layer, rel=0, abs=0)
    assert bench.step_gemm_flops(28) == pytest.approx(69.269232549888e12, rel=1e-15)
    assert bench.step_gemm_flops(1) * 28 == bench.step_gemm_flops(28)


class _FakeEvent:
    def __init__(self, t_ms):
        self.t = t_ms

    def elapsed_time(self, other):
        return other.t - self.t


def test_kernel_breakdown_shares_and_rates():
    launches = [
        ("quant_act", "q", None, 0.0, 4.0e6),        # 4 MB moved
        ("gemm_rowblock", "g", None, 2.0e12, 1.0e6),  # 2 TFLOP
        ("quant_act", "q", None, 0.0, 4.0e6),
        ("gemm_outer", "w", None, 1.0e12, 1.0e6),
    ]
    # two replays, launch durations 1, 2, 1, 4 ms in each
    events = [[_FakeEvent(t) for t in (0.0, 1.0, 3.0, 4.0, 8.0)],
              [_FakeEvent(t) for t in (10.0, 11.0, 13.0, 14.0, 18.0)]]
    kinds = bench.summarize_kernels(launches, events, {}, "measured")
    assert set(kinds) == {"quant_act", "gemm_rowblock", "gemm_outer"}
    assert sum(d["share"] for d in kinds.values()) == pytest.approx(1.0)
    q, g, w = kinds["quant_act"], kinds["gemm_rowblock"], kinds["gemm_outer"]
    assert q["launches"] == 4 and g["launches"] == 2 and w["launches"] == 2
    assert q["share"] == pytest.approx(4 / 16) and g["share"] == pytest.approx(4 / 16)
    assert w["share"] == pytest.approx(8 / 16)
    assert q["avg_us"] == pytest.approx(1000.0)
    assert g["tflops"] == pytest.approx(4.0e12 / 4e-3 / 1e12)     # 1000 TFLOPS
    assert w["tflops"] == pytest.approx(2.0e12 / 8e-3 / 1e12)     # 250 TFLOPS
    assert q["tflops"] is None
    assert q["gbs"] == pytest.approx(16.0e6 / 4e-3 / 1e9)         # 4 GB/s


def test_peaks_measured_file_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk, kind = bench.peaks()
    assert kind == "fallback" and pk == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6539.5, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1376.7}))
    pk, kind = bench.peaks()
    assert kind == "measured" and pk["bf16_tflops_sustained"] == 1376.7


def test_traffic_entries_name_their_launch():
    for kind, (nbytes, what) in bench.NCU_TRAFFIC_BYTES_PER_LAUNCH.items():
        assert kind in ("gemm_rowblock", "gemm_outer", "quant_act", "quant_weight")
        assert nbytes > 0 and "algorithmic" in what and "commit" in what


def test_defaults_keep_the_timing_rules(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    args = bench.parse()
    assert args.gpus == 1 and args.impl == "ours" and args.layers == bench.LAYERS
    assert args.warmup >= 3 and args.steps >= 1


def _wave_model(a, b, threads):
    """Oracle-like timing: rows run in waves of `threads`, plus a fixed cost."""
    calls = []

    def run(rows):
        calls.append(rows)
        return a + b * -(-rows // threads)
    return run, calls


@pytest.mark.parametrize("threads", [1, 8, 16, 112])
def test_calibrate_rows_hits_the_target_on_thread_multiples(threads):
    run, calls = _wave_model(0.05, 0.02, threads)
    rows = bench.calibrate_rows(run, threads, 10.0, max_rows=8192)
    assert (rows % threads == 0 or rows == 8192) and threads <= rows <= 8192
    assert all(r % threads == 0 or r == 8192 for r in calls)   # never below one row per thread
    took = run(rows)
    assert took <= 10.0 + 1e-9
    assert took >= min(10.0 - 0.02, run(8192)) - 1e-9             # within one wave of the target


def test_calibrate_rows_does_not_mistake_idle_threads_for_cheap_rows():
    # 16 threads: 2 and 8 rows cost the same, which must not read as a zero
    # per-row cost (that picked nearly all 8192 rows and a 90 s sample)
    run, _ = _wave_model(0.0, 0.2, 16)
    rows = bench.calibrate_rows(run, 16, 2.0, max_rows=8192)
    assert rows == 160 and run(rows) == pytest.approx(2.0)


def test_calibrate_rows_bounds():
    run, _ = _wave_model(0.0, 1e-4, 8)
    assert bench.calibrate_rows(run, 8, 1e6, max_rows=8192) == 8192     # all rows fit
    run, _ = _wave_model(0.0, 5.0, 8)
    assert bench.calibrate_rows(run, 8, 0.1, max_rows=8192) == 8        # one row per thread at least


def test_reference_arm_prints_one_bounded_line():
    import subprocess

    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1", "--ref-seconds", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    rows = d["config"]["rows_per_gemm"]
    assert rows % d["cpu_baseline"]["cores"] == 0
    assert d["ms_per_step"] < 5000          # about 1 s of oracle work per step was asked for


def test_nvidia_smi_id_follows_cuda_visible_devices():
    assert bench.nvidia_smi_id(0, None) == "0"
    assert bench.nvidia_smi_id(3, "") == "3"
    assert bench.nvidia_smi_id(1, "4,5") == "5"
    assert bench.nvidia_smi_id(0, " GPU-1a2b3c4d-0000 , GPU-ffff") == "GPU-1a2b3c4d-0000"
    assert bench.nvidia_smi_id(2, "7") == "2"


def test_clock_sampler_summarises_reasons_and_clocks(monkeypatch):
    cs = bench.ClockSampler("0")
    cs.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    cs.lines = ["0, 1800, 1965, 900.5, 0x4, Not Active, Not Active, Not Active, Active",
                "0, 1790, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
                "0, 1810, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
                "garbage"]
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    got = cs.stop()
    assert got["sm_mhz"] == 1800 and got["sm_max_mhz"] == 1965 and got["samples"] == 3
    assert got["power_w_max"] == 990.0 and got["reasons"] == ["sw_power_cap"]


def test_clock_rejects_follows_the_timing_rules():
    ok = {"sm_mhz": 1788.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert not bench.clock_rejects(ok)
    assert not bench.clock_rejects({"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": []})
    for bad in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clock_rejects({"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap", bad]})
    # stuck well below max with nothing to explain it: a leftover clock lock
    assert bench.clock_rejects({"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "reasons": []})
    # no sampler: no clock record to check
    assert not bench.clock_rejects({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]})


def test_gpus_must_match_the_launched_world_size(monkeypatch, capsys):
    """--gpus N > 1 without torchrun would time one replica while claiming N:
    both arms refuse it before doing any work."""
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    for impl in ("ours", "reference"):
        monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "2", "--impl", impl])
        assert bench.main() == 2
        assert "WORLD_SIZE=1" in capsys.readouterr().err


def test_roofline_fractions_use_every_denominator():
    pk = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    ceiling = {"8192x8192x8192": {"tflops": 3000.0}, "gate_up_fprop_8192x12288x2048": {"tflops": 2500.0}}
    fr = bench.roofline_fracs(1500.0, pk, "measured", ceiling)
    assert fr["spec_fp8_dense_4500"] == pytest.approx(1500.0 / 4500.0)
    assert fr["2x_measured_bf16_burst"] == pytest.approx(1500.0 / 3200.0)
    assert fr["2x_measured_bf16_sustained"] == pytest.approx(1500.0 / 2800.0)
    assert fr["fp8_library_8192x8192x8192"] == pytest.approx(0.5)
    assert fr["fp8_library_gate_up_fprop_8192x12288x2048"] == pytest.approx(0.6)
    assert "fp8_library_8192x8192x8192" not in bench.roofline_fracs(1.0, pk, "measured", {"error": "x"})
