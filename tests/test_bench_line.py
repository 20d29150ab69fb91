"""The benchmark's JSON line (the driver's contract) assembled from fixed per-rank results on
CPU: every required key is there, the rates are the job's units over the slowest rank's time,
the roofline fraction is achieved over peak, and the line serialises."""
import json
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import workloads as W  # noqa: E402

PEAKS = (6453.7, 1670.0, 1400.0, "measured")


def _pre(ms):
    return {"ms": ms, "e2e_ms": 3 * ms, "launches": 180, "h2d": 134217728, "d2h": 134217728,
            "stages": {"weights_to_16bit": 0.01, "qkv_projection": 0.18, "latent_stencil": 0.25,
                       "latent_attention": 1.39, "out_projection": 0.11}, "calls": 30}


def _dec(ms):
    return {"ms": ms, "launches": 600, "layers": 32, "steps": 200,
            "stages": {"qkv_projection": 0.011, "stencil_append": 0.015,
                       "split_kv_attention": 0.05, "merge": 0.0, "out_projection": 0.011}}


@pytest.mark.parametrize("world", [1, 4])
def test_result_line_contract(world):
    w = W.WORKLOADS[bench.DEFAULT_WORKLOAD]
    pre, dec = _pre(1.95), _dec(0.0656)
    line = bench.result_line(w, world, 30, 5, pre, 1.95, 5.85, dec, 0.0656, PEAKS)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "decode"):
        assert key in line, key
    assert line["config"]["workload"] == w.name and line["n_gpus"] == world
    assert line["steps"] == 30 and line["warmup"] == 5 and line["scaling"] == "weak"
    tokens = w.batch * w.seq
    assert line["value"] == pytest.approx(world * tokens / 1.95e-3)
    assert line["e2e"]["value"] == pytest.approx(world * tokens / 5.85e-3)
    assert line["e2e"]["h2d_bytes_per_step"] == 134217728
    roof = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert roof["achieved"] == pytest.approx(bench.attention_flops(w) / 1.39e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1670.0)
    assert line["gpu_launches"] == 780
    d = line["decode"]
    dw = W.WORKLOADS[bench.DECODE_WORKLOAD]
    assert d["GB/s"] == pytest.approx(bench.decode_bytes(dw) / 0.0656e-3 / 1e9)
    assert d["frac_of_hbm"] == pytest.approx(d["GB/s"] / 6453.7)
    assert d["tokens_per_s"] == pytest.approx(world * dw.batch / 0.0656e-3)
    assert d["steps"] == 200 >= bench.DECODE_MIN_STEPS
    json.loads(json.dumps(line))


def test_result_line_without_decode():
    w = W.WORKLOADS[bench.DEFAULT_WORKLOAD]
    line = bench.result_line(w, 1, 10, 3, _pre(2.0), 2.0, 6.0, None, None, PEAKS)
    assert "decode" not in line and line["gpu_launches"] == 180
