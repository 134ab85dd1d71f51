"""The JSON line bench.py prints, checked on CPU: the measurement itself needs a GPU, so
the timed runs are replaced by stubs that return what a run measures, and the report code
that builds the line runs as it stands.  The reference arm (the oracle on the host) runs
for real on a few bounded steps."""
import json
import sys

import bench
from newton_schulz_hyperball_b200 import workloads as wl

QWEN = [(r, c) for _, r, c in wl.qwen3_1b_shapes(28)]
GPT2 = [(r, c) for _, r, c in wl.gpt2_small_shapes(12)]


def measured(kinds, shp, ms=2.05):
    """A run's measurements as run_cuda returns them (per-kernel ms summed over kp steps)."""
    kp = 20
    n = sum(r * c for r, c in shp)
    return dict(ms=ms, prof={k: (t * kp, c * kp) for k, (t, c) in kinds.items()}, kp=kp,
                launches_per_step=sum(c for _, c in kinds.values()), flags=0,
                clocks={"sm_mhz": 1600, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 200},
                e2e_ms=3.5, h2d=2 * n, d2h=4, n_params=n, shp=shp)


MUONH = {"momentum": (0.22, 1), "norm": (0.01, 1), "gram": (0.445, 5), "poly": (0.376, 5), "update": (0.9, 5),
         "reduce": (0.11, 1), "finalize": (0.02, 2), "exact": (0.008, 1), "apply": (0.11, 1)}
QWEN_MUONH = {"momentum": (2.5, 1), "norm": (0.01, 1), "gram": (12.0, 5), "poly": (9.0, 5), "update": (27.0, 5),
              "reduce": (1.4, 1), "finalize": (0.02, 2), "exact": (0.008, 1), "apply": (1.3, 1)}
ADAMH = {"adam": (0.305, 1), "finalize": (0.02, 2), "exact": (0.008, 1), "apply": (0.08, 1)}


def run_bench(monkeypatch, capsys, argv):
    monkeypatch.setattr(sys, "argv", ["bench.py", *argv])
    assert bench.run() == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, lines
    return json.loads(lines[0])


def check_common(line, steps, warmup):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config"):
        assert k in line, k
    assert line["steps"] == steps and line["warmup"] == warmup >= 3
    assert line["n_gpus"] == 1 and line["scaling"] == "weak" and line["higher_is_better"] is False
    assert line["vs_baseline"] is None
    assert "workload" in line["config"]
    e2e = line["e2e"]
    assert set(e2e) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}


def test_default_line_is_the_qwen3_muonh_set(monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_cuda", lambda *a: measured(QWEN_MUONH, QWEN, ms=55.0))
    line = run_bench(monkeypatch, capsys, ["--steps", "20", "--warmup", "5", "--no-cpu-baseline"])
    check_common(line, 20, 5)
    assert line["metric"] == bench.METRIC and line["unit"] == "ms" and line["value"] == 55.0
    assert line["config"]["workload"].startswith("Qwen3-style") and line["config"]["matrices"] == 196
    assert line["config"]["params"] == 1409286144
    roof = line["roofline"]
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert set(roof) >= {"achieved", "peak", "frac", "traffic"}
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3
    # 20 steps of 55 ms run for over a second: the kernel is held to the sustained peak
    peaks, _ = bench.load_peaks()
    assert roof["peak"] == peaks["bf16_tflops_sustained"]
    # algorithmic NS flops of the set (47.80 TFLOP) over the summed GEMM time of one step
    gemm_ms = 12.0 + 9.0 + 27.0
    assert abs(bench.ns_flops(QWEN) / 1e12 - 47.80) < 0.01
    assert abs(line["ns_tflops"] - bench.ns_flops(QWEN) / (gemm_ms * 1e-3) / 1e12) < 0.1
    # fused streaming bytes: 20 B/elem (momentum 14 with X0's low part, apply 6) over
    # momentum + reduce + apply
    n = 1409286144
    assert abs(line["fused_gbs"] - 20.0 * n / ((2.5 + 1.4 + 1.3) * 1e-3) / 1e9) < 1.0
    assert abs(line["momentum_gbs"] - 14.0 * n / (2.5e-3) / 1e9) < 1.0
    assert line["gpu_launches"] == 22 * 20
    assert line["clocks"]["reasons"] == ["sw_power_cap"]
    assert line["e2e"]["h2d_bytes_per_step"] == 2 * n and line["e2e"]["d2h_bytes_per_step"] == 4


def test_gpt2_line_uses_the_burst_peak(monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_cuda", lambda *a: measured(MUONH, GPT2))
    line = run_bench(monkeypatch, capsys, ["--config", "gpt2", "--steps", "20", "--warmup", "5",
                                           "--no-cpu-baseline"])
    check_common(line, 20, 5)
    peaks, _ = bench.load_peaks()
    assert line["roofline"]["peak"] == peaks["bf16_tflops"]   # 41 ms timed region: burst
    assert line["config"]["matrices"] == 72


def test_adamh_line_carries_every_contract_key(monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_cuda", lambda *a: measured(ADAMH, GPT2))
    line = run_bench(monkeypatch, capsys, ["--optimizer", "adamh", "--steps", "100", "--warmup", "5",
                                           "--no-cpu-baseline"])
    check_common(line, 100, 5)
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    n = sum(r * c for r, c in GPT2)
    # 22 algorithmic bytes per element over the adam kernel's time
    assert abs(roof["achieved"] - 22.0 * n / 0.305e-3 / 1e9) < 1.0
    assert line["gpu_launches"] == 5 * 100


def test_reference_arm_runs_the_oracle_and_reports_what_it_timed(monkeypatch, capsys):
    line = run_bench(monkeypatch, capsys, ["--impl", "reference", "--config", "gpt2", "--steps", "4",
                                           "--warmup", "3"])
    check_common(line, 4, 3)
    assert line["impl"] == "reference" and line["dtype"] == "f64"
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"] > 0
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    # ms_per_step is the time of a timed step (one matrix); value extrapolates it to the set
    assert line["extrapolated"] is True and line["ms_per_step"] < line["value"]
    # warm-up takes matrices 0..2, the four timed steps matrices 3, 4, 5 and 6 (layer 1's Wq)
    assert "4 timed steps" in cpu["sample"] and "h1.wq" in cpu["sample"]


def test_warmup_below_three_is_raised_to_three(monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_cuda", lambda *a: measured(QWEN_MUONH, QWEN, ms=55.0))
    line = run_bench(monkeypatch, capsys, ["--steps", "10", "--warmup", "1", "--no-cpu-baseline"])
    assert line["warmup"] == 3


def test_cpu_sample_extrapolation_is_exact_for_identical_layers():
    """The Qwen3-style set is 28 copies of one layer: its sample (layer 0) scales by 28."""
    args = type("A", (), {"config": "qwen3", "layers": 0, "tile": 256})()
    w = bench.make_workload(args)
    idx, _ = bench.cpu_sample_plan(w)
    full = sum(bench.unit_cost(w, i) for i in range(len(w.shapes)))
    part = sum(bench.unit_cost(w, i) for i in idx)
    assert abs(full / part - 28.0) < 1e-9
