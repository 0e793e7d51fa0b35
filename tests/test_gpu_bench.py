"""The benchmark's JSON line on a B200: a short run of the default (8-window
encoder) workload and of the verify step through bench.main, checked for
every key the measurement contract asks for and for values that hang
together (the roofline's achieved figure over its peak is its fraction; the
end-to-end bytes are the step's input and output; the dominant kernel's
launches are this library's)."""
import json

import pytest

pytestmark = pytest.mark.gpu


def run_bench(capsys, *args):
    import bench
    assert bench.main(list(args)) == 0
    lines = [ln for ln in capsys.readouterr().out.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1, "bench prints exactly one JSON line"
    return json.loads(lines[0])


def check_common(d, steps, warmup):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["gpu_launches"] > 0
    r = d["roofline"]
    assert r["bound"] in ("tensor", "hbm") and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9 and 0 < r["frac"] < 2
    c = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(c)


def test_default_line(capsys):
    d = run_bench(capsys, "--steps", "5", "--warmup", "3", "--cpu-seconds", "1", "--e2e-steps", "5")
    check_common(d, 5, 3)
    assert d["config"]["workload"].startswith("windows8")
    assert d["unit"] == "TFLOP/s" and d["roofline"]["bound"] == "tensor" and d["roofline"]["unit"] == "TFLOP/s"
    e = d["e2e"]
    assert e["unit"] == d["unit"] and e["value"] > 0
    assert e["h2d_bytes_per_step"] == e["d2h_bytes_per_step"] == 8 * 1500 * 1280 * 2
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    assert set(d["kernels"]) == {"qkv_gemm", "flash_attn"}


def test_verify_line(capsys):
    d = run_bench(capsys, "--workload", "verify", "--steps", "50", "--warmup", "5", "--skip-cpu-baseline",
                  "--e2e-steps", "20")
    check_common(d, 50, 5)
    assert d["roofline"]["bound"] == "hbm" and d["roofline"]["unit"] == "GB/s"
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
