"""bench.py's JSON line from synthetic measurements (no GPU): every key the
benchmark contract names is present with the right type, the rates follow
from the timings, and the line serializes."""
import json
import types

import pytest


def _measurements(e2e=True, extras=True):
    r = {"ms_total": 300 * 3.34, "ms_quant": 0.080, "ms_attn": 3.26,
         "clocks": {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                    "samples": 7},
         "e2e_ms": 3.38 if e2e else None, "attn_launches": 2,
         "rollouts": None, "matrix": None, "dequant": None}
    if extras:
        r["rollouts"] = [{"workload": "w", "chunks_per_s": 11.0, "frac": 0.66}]
        r["matrix"] = [{"workload": "m", "us_per_launch": 42.0}]
        r["dequant"] = {"kernel": "d", "us_per_launch": 27.0}
        r["rope"] = {"workload": "r", "table_us": 8.0,
                     "rope": {"us_per_launch": 17.0, "frac": 0.77},
                     "quantize_rope": {"us_per_launch": 80.0, "unfused_us": 75.0}}
    return r


@pytest.mark.parametrize("world", [1, 4])
def test_line_has_the_contract_keys(world):
    import bench
    args = types.SimpleNamespace(steps=300, warmup=10)
    line = bench.build_line(args, _measurements(), world, {}, "fallback")
    for k, t in (("metric", str), ("value", float), ("unit", str), ("n_gpus", int),
                 ("steps", int), ("warmup", int), ("ms_per_step", float),
                 ("higher_is_better", bool), ("scaling", str), ("dtype", str), ("data", str),
                 ("config", dict), ("roofline", dict), ("e2e", dict), ("gpu_launches", int),
                 ("clocks", dict)):
        assert isinstance(line[k], t), k
    assert line["vs_baseline"] is None and line["scaling"] == "weak" and line["n_gpus"] == world
    assert "workload" in line["config"]
    rf = line["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"])
    assert rf["frac_burst"] == pytest.approx(rf["achieved"] / bench.FALLBACK_PEAKS["bf16_tflops"])
    assert rf["frac_sustained"] == pytest.approx(
        rf["achieved"] / bench.FALLBACK_PEAKS["bf16_tflops_sustained"])
    assert rf["achieved"] == pytest.approx(bench.attn_flops() / 3.26e-3 / 1e12)
    # whole-job rate: all ranks' work over the (slowest rank's) time
    assert line["value"] == pytest.approx(bench.attn_flops() * 300 * world / (300 * 3.34e-3) / 1e12)
    e = line["e2e"]
    assert e["unit"] == line["unit"] and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert line["gpu_launches"] == 300 * 3
    for k in ("rollouts", "matrix_quantize", "dequantize", "quantize", "attention", "rope"):
        assert k in line
    json.dumps(line)


def test_line_without_optional_parts():
    import bench
    args = types.SimpleNamespace(steps=20, warmup=3)
    line = bench.build_line(args, _measurements(e2e=False, extras=False), 1, {}, "fallback")
    for k in ("e2e", "rollouts", "matrix_quantize", "dequantize", "rope"):
        assert k not in line
    json.dumps(line)


def test_cpu_baseline_only_in_one_gpu_runs():
    import bench
    on = types.SimpleNamespace(no_cpu_baseline=False)
    off = types.SimpleNamespace(no_cpu_baseline=True)
    assert bench.wants_cpu_baseline(on, 1)
    assert not bench.wants_cpu_baseline(on, 2)
    assert not bench.wants_cpu_baseline(off, 1)


@pytest.mark.parametrize("steps,basis", [(20, "burst"), (200, "burst"), (600, "sustained")])
def test_attention_peak_follows_the_timed_region(steps, basis):
    """A kernel timed over a short region (a driver run of 20 steps is ~66 ms)
    is held to the burst bf16 peak; one timed over seconds to the sustained."""
    import bench
    peaks = {"hbm_gbs": 6551.4, "bf16_tflops": 1618.2, "bf16_tflops_sustained": 1377.3}
    r = _measurements()
    r["ms_total"] = steps * 3.29
    line = bench.build_line(types.SimpleNamespace(steps=steps, warmup=5), r, 1, peaks,
                            "measured")
    rf = line["roofline"]
    want = peaks["bf16_tflops"] if basis == "burst" else peaks["bf16_tflops_sustained"]
    assert rf["peak"] == want and basis in rf["peak_source"]
    assert rf["frac"] == pytest.approx(rf["achieved"] / want)
    assert rf["frac_burst"] == pytest.approx(rf["achieved"] / 1618.2)


def test_reference_line_matches_our_config(monkeypatch, capsys):
    """--impl reference reports our arm's metric, unit and config, the measured
    seconds of each timed sample as ms_per_step, and the extrapolation apart."""
    import bench

    class FakeSample:
        def __init__(self, rows):
            pass

        def run(self):
            return 0.003, 0.2, 0.19, 0.1, 0.25

        def entry(self, value, ta, tq):
            return {"value": value, "unit": "TFLOP/s", "cores": 8, "kind": "oracle",
                    "sample": "s"}

    monkeypatch.setattr(bench, "OracleSample", FakeSample)
    monkeypatch.delenv("RANK", raising=False)
    args = types.SimpleNamespace(ref_rows=32, warmup=3, steps=4, gpus=1)
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip())
    ours = bench.build_line(types.SimpleNamespace(steps=4, warmup=3), _measurements(), 1, {},
                            "fallback")
    assert line["impl"] == "reference" and line["config"] == ours["config"]
    assert line["metric"] == ours["metric"] and line["unit"] == ours["unit"]
    assert line["ms_per_step"] == pytest.approx(250.0)
    assert line["extrapolated"]["extrapolated"] is True
    assert line["e2e"]["h2d_bytes_per_step"] == 0
