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
    assert rf["achieved"] == pytest.approx(bench.attn_flops() / 3.26e-3 / 1e12)
    # whole-job rate: all ranks' work over the (slowest rank's) time
    assert line["value"] == pytest.approx(bench.attn_flops() * 300 * world / (300 * 3.34e-3) / 1e12)
    e = line["e2e"]
    assert e["unit"] == line["unit"] and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert line["gpu_launches"] == 300 * 3
    for k in ("rollouts", "matrix_quantize", "dequantize", "quantize", "attention"):
        assert k in line
    json.dumps(line)


def test_line_without_optional_parts():
    import bench
    args = types.SimpleNamespace(steps=20, warmup=3)
    line = bench.build_line(args, _measurements(e2e=False, extras=False), 1, {}, "fallback")
    for k in ("e2e", "rollouts", "matrix_quantize", "dequantize"):
        assert k not in line
    json.dumps(line)


def test_cpu_baseline_only_in_one_gpu_runs():
    import bench
    on = types.SimpleNamespace(no_cpu_baseline=False)
    off = types.SimpleNamespace(no_cpu_baseline=True)
    assert bench.wants_cpu_baseline(on, 1)
    assert not bench.wants_cpu_baseline(on, 2)
    assert not bench.wants_cpu_baseline(off, 1)
