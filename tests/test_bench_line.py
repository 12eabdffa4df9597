"""bench.py's JSON line: every key the benchmark contract asks for, with the
whole-job throughput and roofline arithmetic, built from given times (no
GPU: the GPU arm calls the same function with its measurements)."""

import importlib.util
import json
import os

import pytest

import fqa_synth as synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("world", [1, 8])
def test_step_line_has_the_contract_keys(world):
    b = _bench()
    w = synth.workload("kontext_n8704")
    pk = {"hbm_gbs": 6559.0, "bf16_tflops": 1656.2}
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5}
    cpu = {"value": 0.05, "unit": "TFLOP/s", "cores": 16, "kind": "oracle", "sample": "s"}
    line = b.step_line(w, world, 100, 20, ms_per_step=0.8, attn_ms=0.744, quant_ms=0.058, bf16_ms=1.05,
                       e2e_ms=3.15, h2d=160432128, d2h=53477376, clocks=clocks, probe=None, cpu=cpu,
                       traffic=98970112, pk=pk, pk_kind="measured")
    json.dumps(line)                                   # one JSON line
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
                "clocks", "cpu_baseline"):
        assert key in line, key
    assert line["metric"] == b.METRIC and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["n_gpus"] == world and line["steps"] == 100 and line["warmup"] == 20
    assert line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["config"]["workload"] == "kontext_n8704"
    assert line["value"] == pytest.approx(w.flops * world / 0.8e-3 / 1e12)
    r = line["roofline"]
    assert set(("bound", "achieved", "peak", "unit", "frac", "traffic")) <= set(r)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["traffic"] == 98970112
    assert r["peak"] == pytest.approx(2 * 1656.2)
    assert r["achieved"] == pytest.approx(w.flops / 0.744e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    e = line["e2e"]
    assert e["unit"] == "TFLOP/s" and e["h2d_bytes_per_step"] == 160432128 and e["d2h_bytes_per_step"] == 53477376
    assert e["value"] == pytest.approx(w.flops * world / 3.15e-3 / 1e12)
    assert line["gpu_launches"] == 200
    assert line["quantizer"]["gbs"] == pytest.approx(9 * w.B * w.H * w.N * w.d / 0.058e-3 / 1e9)
    assert line["cpu_baseline"] is cpu and line["clocks"] is clocks
