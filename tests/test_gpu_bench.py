"""bench.py's native arm on a B200: one short run prints one JSON line with
every key of the benchmark contract, in the units and relations the
contract fixes (the roofline's kernel time inside the step time, the
instrumented launches inside the timed region, the launch count, the
end-to-end figure's byte counts)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_native_arm_json_line():
    steps, warmup = 8, 3
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", str(steps), "--warmup", str(warmup),
           "--no-per-config", "--e2e-steps", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup
    assert d["unit"] == "TOPS" and d["dtype"] == "int8" and d["higher_is_better"] is True
    assert d["scaling"] == "weak" and d["value"] > 0 and d["config"]["workload"].startswith("mlp_up_1024")
    # two kernels of the library per step: the quantizer and the GEMM
    assert d["gpu_launches"] == 2 * steps
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TOPS" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    # the GEMM's live launch time lies inside the step it belongs to
    assert 0 < r["ms_per_launch"] < d["ms_per_step"]
    # a short timed region is compared with the burst peak, a region of a second or more with the sustained one
    assert r["peak_kind"] == "burst" and r["peak"] == r["burst_peak"] > r["sustained_peak"]
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["unit"] == "TOPS"
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 4096 * 3072 * 2 and e["d2h_bytes_per_step"] == 4096 * 12288 * 2
    assert 0 < e["value"] < d["value"]
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]


def test_native_arm_per_config_table():
    """The per-configuration table of the default bench line: every DiT
    layer shape timed, with the paper's accuracy metric beside it (cosine
    similarity against the float64 product, no NaN in the output)."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "4", "--warmup", "3", "--e2e-steps", "0",
           "--no-cpu-baseline"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=1200, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.strip().startswith("{")][-1])
    rows = d["per_config"]["configs"]
    assert [r["workload"] for r in rows] == ["qkv_768", "mlp_up_1024", "mlp_down_1024", "sweep_qkv", "sweep_out",
                                             "sweep_up", "sweep_down"]
    for r in rows:
        assert r["gemm_us"] > 0 and r["gemm_tops"] > 0, r["workload"]
        acc = r["accuracy"]
        assert acc["nan_outputs"] == 0, r["workload"]
        # with x20 outlier channels (MLP up) the per-token quantization itself costs ~1e-3 of cosine
        assert acc["cosine_vs_fp64"] > (0.99 if acc["against"] == "unquantized operands" else 0.9999), r
        if r["workload"] != "mlp_down_1024":
            assert r["linear_us"] > 0 and r["quant_gbs"] > 0, r["workload"]
