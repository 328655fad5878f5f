"""bench.py's reference arm on the CPU: it runs the oracle on a bounded
sample and prints one JSON line with the keys the benchmark contract asks
for (the native arm needs a GPU and is exercised by the GPU runs)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches"}


@pytest.mark.parametrize("args", [["--workload", "tiny"], ["--workload", "tiny", "--format", "fp8"],
                                  ["--workload", "dit_block_1024"]], ids=["int8", "fp8", "block"])
def test_reference_arm_json(args):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3", "--warmup", "3"]
    out = subprocess.run(cmd + args, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 3 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["gpu_launches"] == 0


def test_warmup_below_three_is_rejected():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "3", "--warmup", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("workload,kind", [("mlp_up_1024", "two-kernel"), ("mlp_up_1024", "fp8"),
                                           ("dit_block_1024", "block")])
def test_traffic_files_only_count_for_the_sources_they_were_taken_on(monkeypatch, workload, kind):
    """The committed ncu traffic of a bench line's dominant kernel is reported
    only while the kernel sources hash to the value recorded with it."""
    b = _bench_module()
    with open(os.path.join(ROOT, "profiles", f"dram_{kind}_{workload}.json")) as fh:
        rec = json.load(fh)
    assert rec["dram_bytes_per_launch"] > 0
    monkeypatch.setattr(b, "gemm_source_hash", lambda: rec["gemm_source_hash"])
    assert b.ncu_traffic(workload, kind)["dram_bytes_per_launch"] == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(b, "gemm_source_hash", lambda: "0" * 16)
    assert b.ncu_traffic(workload, kind) is None


def test_roofline_peak_follows_the_timed_region():
    """The tensor peak a roofline fraction is taken against: twice the
    measured bf16 figure, the burst one for a timed region under a second,
    the sustained one for a second or more; the other fractions beside it."""
    b = _bench_module()
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "measured"}
    short = b.tensor_peak(peaks, 2.4)
    assert short["kind"] == "burst" and short["peak"] == 3200.0
    long_ = b.tensor_peak(peaks, 1500.0)
    assert long_["kind"] == "sustained" and long_["peak"] == 2800.0
    assert b.tensor_peak(peaks, 1000.0)["kind"] == "sustained"
    det = short["detail"](1600.0)
    assert det["frac_of_burst_peak"] == 0.5 and det["frac_of_sustained_peak"] == 1600.0 / 2800.0
    assert abs(det["frac_of_spec_4p5"] - 1600.0 / 4500.0) < 1e-12
    assert "2.4 ms" in det["peak_source"] and "burst" in det["peak_source"]


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the round-end scaling run launches it (torchrun, two ranks
    on this host), the reference arm's rank 0 alone runs and prints its one
    line; the other rank exits 0 without work."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "3", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
