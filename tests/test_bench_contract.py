"""The JSON line bench.py prints, checked on CPU: the measurement itself needs a GPU, so
the timed runs are replaced by stubs that return what a run measures, and the report code
that builds the line runs as it stands.  The reference arm (the oracle on the host) runs
for real on one bounded step."""
import json
import sys

import bench
from newton_schulz_hyperball_b200 import workloads as wl

SHP = [(r, c) for _, r, c in wl.gpt2_small_shapes(12)]
N_PARAMS = sum(r * c for r, c in SHP)


def measured(kinds):
    """A run's measurements as run_cuda / run_adamh return them (per-kernel ms summed over kp steps)."""
    kp = 50
    return dict(ms=2.05, prof={k: (ms * kp, n * kp) for k, (ms, n) in kinds.items()}, kp=kp,
                launches_per_step=sum(n for _, n in kinds.values()), flags=0,
                clocks={"sm_mhz": 1600, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 20},
                e2e_ms=3.5, h2d=2 * N_PARAMS, d2h=4, n_params=N_PARAMS, shp=SHP)


MUONH = {"momentum": (0.22, 1), "norm": (0.01, 1), "gram": (0.445, 5), "poly": (0.376, 5), "update": (0.9, 5),
         "reduce": (0.11, 1), "finalize": (0.02, 2), "exact": (0.008, 1), "apply": (0.11, 1)}
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


def test_muonh_line_carries_every_contract_key(monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_cuda", lambda *a: measured(MUONH))
    line = run_bench(monkeypatch, capsys, ["--steps", "200", "--warmup", "10", "--no-cpu-baseline"])
    check_common(line, 200, 10)
    assert line["metric"] == bench.METRIC and line["unit"] == "ms" and line["value"] == 2.05
    roof = line["roofline"]
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert set(roof) >= {"achieved", "peak", "frac", "traffic"}
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3
    # algorithmic NS flops of the set over the summed GEMM time of one step
    gemm_ms = 0.445 + 0.376 + 0.9
    assert abs(line["ns_tflops"] - bench.ns_flops(SHP) / (gemm_ms * 1e-3) / 1e12) < 0.1
    assert line["gpu_launches"] == 22 * 200
    assert line["clocks"]["reasons"] == ["sw_power_cap"]
    assert line["e2e"]["h2d_bytes_per_step"] == 2 * N_PARAMS and line["e2e"]["d2h_bytes_per_step"] == 4


def test_adamh_line_carries_every_contract_key(monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_adamh", lambda *a: measured(ADAMH))
    line = run_bench(monkeypatch, capsys, ["--optimizer", "adamh", "--steps", "100", "--warmup", "5",
                                           "--no-cpu-baseline"])
    check_common(line, 100, 5)
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    # 22 algorithmic bytes per element over the adam kernel's time
    assert abs(roof["achieved"] - 22.0 * N_PARAMS / 0.305e-3 / 1e9) < 1.0
    assert line["gpu_launches"] == 5 * 100


def test_reference_arm_runs_the_oracle(monkeypatch, capsys):
    line = run_bench(monkeypatch, capsys, ["--impl", "reference", "--steps", "1", "--warmup", "1"])
    check_common(line, 1, 3)
    assert line["impl"] == "reference" and line["dtype"] == "f64"
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"] > 0
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0


def test_warmup_below_three_is_raised_to_three(monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_cuda", lambda *a: measured(MUONH))
    line = run_bench(monkeypatch, capsys, ["--steps", "10", "--warmup", "1", "--no-cpu-baseline"])
    assert line["warmup"] == 3
