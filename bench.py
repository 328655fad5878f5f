"""Benchmark of the W8A8 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

One step is one W8A8 linear layer (per-token quantization -> tcgen05 int8
GEMM -> dequant + bias epilogue -> bf16) over one token batch of the
workload, by default the 1024px DiT MLP up-projection (M=4096 tokens,
K=3072, N=12288).  Inputs are seeded synthetic data resident in HBM; the
step cycles through enough buffer sets (activations, weights, workspace,
output) that their combined footprint is several times the 126 MB L2, so
every step reads its operands from HBM.

Printed (rank 0, one JSON line): whole-job int8 TOPS (2*M*N*K per step,
summed over ranks, divided by the max over ranks of the device time),
the GEMM kernel's roofline against the int8 tensor peak, the quantizer's
GB/s, the end-to-end figure through the public API with host buffers, the
CPU oracle timed on a bounded sample, SM clocks sampled during the timed
region, and context (bf16 torch.matmul and the dequantize-then-bf16-GEMM
path on the same shape).

Multi-GPU (torchrun, one process per GPU): tokens are independent, so each
rank runs its own token batch against a replicated weight with no
data-path collective (weak scaling); torch.distributed is used only for the
barrier and the max over ranks of the timed region.

--impl reference times the CPU oracle (the plain C reference of the method)
on the host cores instead, on a bounded row sample per step, and prints
the same metric for it.

--format fp8 runs the FP8 (OCP E4M3) variant of the same layer instead
(w8a8_linear_fp8: E4M3 quantizer, tcgen05 kind::f8f6f4 GEMM, the same
epilogue), the paper's comparison baseline, with its own metric line; its
context adds the library FP8 GEMM (torch._scaled_mm, row-wise scales).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused W8A8 linear TOPS and % of B200 dense INT8 peak per M×N×K; quantizer GB/s"
METRIC_BLOCK = "W8A8 DiT-block linear chain TOPS (four linears recorded as one CUDA graph)"
METRIC_FP8 = "fused W8A8 linear, FP8 (E4M3) variant: TFLOPS and % of B200 dense FP8 peak per M×N×K"
L2_BYTES = 126 * 1024 * 1024
NOMINAL_INT8_OVER_BF16 = 2.0     # 4.5 POPS dense int8 / 2.25 PFLOP/s dense bf16 (B200 datasheet)
# dense fp8 is 4.5 PFLOP/s too: the same ratio
SPEC_INT8_POPS = 4500.0          # B200 dense int8, TOPS
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
GEMM_SOURCES = ["w8a8_int8_gemm_b200/csrc/gemm_sm100.cu", "w8a8_int8_gemm_b200/csrc/sm100_ptx.cuh",
                "w8a8_int8_gemm_b200/csrc/quant_row.cuh", "w8a8_int8_gemm_b200/csrc/api.cu"]


# ---------------------------------------------------------------- helpers


def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_token_rows(M: int, rank: int) -> slice:
    """Rows of the (seeded) token stream that rank `rank` processes: every
    rank runs its own batch of M tokens (weak scaling); tokens are
    independent, so no rank needs another rank's data."""
    return slice(rank * M, (rank + 1) * M)


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the timed region's wall time)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def tensor_peak(peaks: dict, region_ms: float, fmt: str = "int8") -> dict:
    """The dense int8 (or fp8) tensor peak a kernel's roofline fraction is
    taken against: the measured bf16 cuBLAS figure times the nominal dense
    int8/bf16 (fp8/bf16) ratio of 2, the burst figure for a kernel timed in a
    region shorter than a second, the sustained (power-capped) one for a
    region of a second or more.  detail(achieved) gives the fractions of
    both and of the 4.5 POPS (PFLOP/s) spec."""
    sustained = region_ms >= 1000.0
    burst_peak = peaks["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    sus_peak = peaks["bf16_tflops_sustained"] * NOMINAL_INT8_OVER_BF16
    peak = sus_peak if sustained else burst_peak
    which = "sustained" if sustained else "burst"
    src = (f"{peaks['source']} {which} bf16 "
           f"{peaks['bf16_tflops_sustained'] if sustained else peaks['bf16_tflops']} TFLOP/s x "
           f"{NOMINAL_INT8_OVER_BF16} (nominal dense {fmt}/bf16 ratio), {which} because the timed region "
           f"lasted {region_ms:.1f} ms ({'>=' if sustained else '<'} 1 s)")

    def detail(achieved: float) -> dict:
        return {"peak_kind": which, "peak_source": src, "frac_of_burst_peak": achieved / burst_peak,
                "frac_of_sustained_peak": achieved / sus_peak, "frac_of_spec_4p5": achieved / SPEC_INT8_POPS,
                "burst_peak": burst_peak, "sustained_peak": sus_peak}

    return {"peak": peak, "kind": which, "detail": detail}


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, path_kind: str) -> dict | None:
    """DRAM bytes per launch of the step's dominant kernel from the committed
    ncu summary, if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"dram_{path_kind}_{workload}.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return None
    if d.get("gemm_source_hash") != gemm_source_hash():
        return None
    return d


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, RuntimeError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= len(self.FIELDS) - 1]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        pw = [float(r[2]) for r in rows if r[2].replace(".", "", 1).isdigit()]
        loaded = [s for s, p in zip(sm, pw) if p > 300] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------ CPU oracle


class OracleWork:
    """The workload prepared once for the CPU oracle: the weight quantized by
    the oracle, and a pool of token rows.  sample(rows, cols, i) runs the
    whole layer (quantize, exact GEMM, epilogue) for `rows` tokens against
    the first `cols` output channels and returns its wall time."""

    def __init__(self, wl: workloads.Workload, pool_rows: int = 512, fp8: bool = False):
        import oracle
        self.o = oracle
        self.wl = wl
        self.fp8 = fp8
        self.pool = min(pool_rows, wl.M)
        if fp8 and wl.kind != "linear":
            raise SystemExit("the FP8 variant runs on the linear-layer workloads")
        if wl.kind == "linear":
            d = workloads.make(wl, rows=slice(0, self.pool))
            self.x = d["x"]
            quantize_weight = oracle.quantize_weight_fp8 if fp8 else oracle.quantize_weight
            self.wq, self.sw = quantize_weight(d["w"])
            self.bias = d["bias"]
        else:
            d = workloads.make(wl)
            self.xq, self.sa = d["xq"][:self.pool], d["scale_a"][:self.pool]
            self.wq, self.sw, self.bias = d["wq"], d["scale_w"], d["bias"]
        self.threads = oracle.default_threads()

    def sample(self, rows: int, cols: int, i: int = 0) -> float:
        r0 = (i * rows) % max(1, self.pool - rows + 1)
        sl = slice(r0, r0 + rows)
        wq, sw, bias = self.wq[:cols], self.sw[:cols], self.bias[:cols]
        t0 = time.perf_counter()
        if self.fp8:
            xq, sa = self.o.quantize_act_fp8(self.x[sl])
            self.o.epilogue_fp8(self.o.gemm_fp8(xq, wq), sa, sw, bias)
        elif self.wl.kind == "linear":
            self.o.linear(self.x[sl], wq, sw, bias)
        else:
            self.o.epilogue(self.o.gemm_i64(self.xq[sl], wq), self.sa[sl], sw, bias)
        return time.perf_counter() - t0


def size_sample(work: OracleWork, seconds: float) -> tuple[int, int]:
    """Rows x columns of one oracle sample taking about `seconds`."""
    wl = work.wl
    t1 = max(work.sample(1, wl.N), 1e-6)
    rows = int(seconds / t1)
    if rows >= 1:
        return min(rows, work.pool), wl.N
    cols = max(8, int(wl.N * seconds / t1) // 8 * 8)
    return 1, min(cols, wl.N)


def cpu_baseline(wl: workloads.Workload, budget_s: float = 12.0, fp8: bool = False) -> dict:
    work = OracleWork(wl, fp8=fp8)
    rows, cols = size_sample(work, budget_s)
    dt = work.sample(rows, cols)
    ops = 2.0 * rows * cols * wl.K
    return {"value": ops / dt / 1e12, "unit": "TFLOPS" if fp8 else "TOPS", "cores": work.threads, "kind": "oracle",
            "sample": f"{rows} of {wl.M} tokens x {cols} of {wl.N} output channels of {wl.name} "
                      f"(K={wl.K}): whole layer (quantize + exact GEMM + epilogue), {dt:.2f} s",
            "seconds": dt}


def run_reference(args, wl) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    fp8 = args.format == "fp8"
    work = OracleWork(wl, fp8=fp8)
    budget = 120.0
    rows, cols = size_sample(work, budget / max(1, args.steps + args.warmup))
    for i in range(args.warmup):
        work.sample(rows, cols, i)
    total = 0.0
    for i in range(args.steps):
        total += work.sample(rows, cols, args.warmup + i)
    ops = 2.0 * rows * cols * wl.K * args.steps
    value = ops / total / 1e12
    sample = (f"{rows} of {wl.M} tokens x {cols} of {wl.N} output channels of {wl.name} per step "
              f"(K={wl.K}), whole layer")
    unit = "TFLOPS" if fp8 else "TOPS"
    line = {"impl": "reference", "metric": METRIC_FP8 if fp8 else METRIC, "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64" if fp8 else "int64",
            "data": "synthetic", "config": wl_config(wl),
            "cpu_baseline": {"value": value, "unit": unit, "cores": work.threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def wl_config(wl) -> dict:
    return {"workload": f"{wl.name}: {wl.note}", "M": wl.M, "N": wl.N, "K": wl.K,
            "l2": "rotating buffer sets, combined footprint > 3x L2"}


# ------------------------------------------------------------- native arm


def run_native(args, wl) -> None:
    import w8a8_int8_gemm_b200 as w8

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    # One dedicated stream (graph capture cannot use the legacy default stream).
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        _run_native_on(args, wl, w8, rank, world, local, dev, stream)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def _run_native_on(args, wl, w8, rank, world, local, dev, stream) -> None:
    # seeded inputs; each rank has its own token batch, the weight is replicated
    M, N, K = wl.M, wl.N, wl.K
    if wl.kind != "linear":
        raise SystemExit(f"workload {wl.name} gives int8 codes; bench the linear-layer workloads")
    fp8 = args.format == "fp8"
    if fp8 and args.path == "fused":
        raise SystemExit("the one-kernel fused path is int8 only")
    # the entry points of the chosen format (codes are int8, or E4M3 bytes)
    code_dtype = torch.uint8 if fp8 else torch.int8
    quantize_weight = w8.w8a8_quantize_weight_fp8 if fp8 else w8.w8a8_quantize_weight
    quantize_act = w8.w8a8_quantize_act_fp8 if fp8 else w8.w8a8_quantize_act
    gemm = w8.w8a8_gemm_fp8 if fp8 else w8.w8a8_gemm
    linear = w8.w8a8_linear_fp8 if fp8 else w8.w8a8_linear
    d = workloads.make(wl, rows=rank_token_rows(M, rank))
    w32 = torch.from_numpy(d["w"]).to(dev)
    x_host = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16)
    bias = torch.from_numpy(d["bias"].view(np.int16)).view(torch.bfloat16).to(dev)
    wq0, sw = quantize_weight(w32)
    del w32

    set_bytes = M * K * 2 + N * K + M * K + M * N * 2 + 4 * M
    nsets = max(2, int(np.ceil(3 * L2_BYTES / set_bytes)))
    sync_words = w8.w8a8_linear_sync_words(M)
    sets = []
    for i in range(nsets):
        x = x_host.to(dev) if i == 0 else torch.roll(sets[0]["x"], shifts=i, dims=0)
        sets.append({"x": x.contiguous(), "wq": wq0 if i == 0 else wq0.clone(),
                     "xq": torch.empty((M, K), dtype=code_dtype, device=dev),
                     "sa": torch.empty((M,), dtype=torch.float32, device=dev),
                     "sync": torch.zeros((sync_words,), dtype=torch.int32, device=dev),
                     "out": torch.empty((M, N), dtype=torch.bfloat16, device=dev)})

    def step_fused(i):
        s = sets[i % nsets]
        w8.w8a8_linear_fused(s["x"], s["wq"], sw, bias, out=s["out"], ws_xq=s["xq"], ws_scale_a=s["sa"],
                             ws_sync=s["sync"], stream=stream)

    def step_linear(i):
        s = sets[i % nsets]
        linear(s["x"], s["wq"], sw, bias, out=s["out"], ws_xq=s["xq"], ws_scale_a=s["sa"], stream=stream)

    def step_quant(i):
        s = sets[i % nsets]
        quantize_act(s["x"], xq=s["xq"], scale_a=s["sa"], stream=stream)

    def step_gemm(i):
        s = sets[i % nsets]
        gemm(s["xq"], s["wq"], s["sa"], sw, bias, out=s["out"], stream=stream)

    step = step_fused if args.path == "fused" else step_linear
    launches_per_step = 1 if args.path == "fused" else 2

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if w8.w8a8_read_device_error() != 0:
        raise SystemExit("a kernel wait timed out during warm-up")

    def capture(fn, n):
        """A CUDA graph of n back-to-back calls of fn (cycling the buffer sets)."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            for i in range(n):
                fn(i)
        return g

    # The timed region replays CUDA graphs of the step (the host launch cost of
    # the Python binding is not part of the layer); exactly K steps run.  Its
    # last G_inst steps replay an instrumented graph that brackets every
    # launch of the dominant kernel (the GEMM) with CUDA events, which gives
    # that kernel's duration live inside the timed region at any step count.
    # Those steps launch the GEMM plainly, without the programmatic overlap
    # the events would break, so they are kept to a quarter of the region
    # (at least one step, at most G).
    G = nsets * max(1, 32 // nsets)
    G_inst = max(1, min(G, args.steps // 4))
    inst_ev = [(torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)) for _ in range(G_inst)]

    def step_instrumented(i):
        if args.path == "fused":
            inst_ev[i][0].record(stream)
            step_fused(i)
            inst_ev[i][1].record(stream)
        else:
            step_quant(i)
            inst_ev[i][0].record(stream)
            step_gemm(i)
            inst_ev[i][1].record(stream)

    n_main, n_tail = divmod(args.steps - G_inst, G)
    g_main = capture(step, G) if n_main else None
    g_tail = capture(step, n_tail) if n_tail else None
    g_inst = capture(step_instrumented, G_inst)
    for g in (g_main, g_tail, g_inst):
        if g is not None:
            g.replay()
    torch.cuda.synchronize(dev)

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    start.record(stream)
    for _ in range(n_main):
        g_main.replay()
    if g_tail is not None:
        g_tail.replay()
    g_inst.replay()
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dev)
    code = w8.w8a8_read_device_error()
    if code != 0:
        raise SystemExit(f"a kernel wait timed out in the timed region (site {code})")
    live_kernel_ms = statistics.fmean(a.elapsed_time(b) for a, b in inst_ev)

    ms_step = elapsed_ms / args.steps
    ops = 2.0 * M * N * K
    value = ops * world / (ms_step * 1e-3) / 1e12

    def graph_ms(fn, reps):
        """Mean ms per call of fn: a graph of G calls, timed with CUDA events."""
        try:
            g = capture(fn, G)
        except RuntimeError as exc:  # e.g. a launch kind the graph cannot hold
            print(f"[bench] could not capture {fn.__name__}: {exc}", file=sys.stderr)
            torch.cuda.synchronize(dev)
            return None
        g.replay()
        a_ev = torch.cuda.Event(enable_timing=True)
        b_ev = torch.cuda.Event(enable_timing=True)
        a_ev.record(stream)
        for _ in range(reps):
            g.replay()
        b_ev.record(stream)
        torch.cuda.synchronize(dev)
        return a_ev.elapsed_time(b_ev) / (reps * G)

    peaks = measured_peaks()
    quant_bytes = 3 * M * K + 4 * M
    kernel_ms = live_kernel_ms
    kernel_tops = ops / (kernel_ms * 1e-3) / 1e12
    roof_peak = tensor_peak(peaks, elapsed_ms, "fp8" if fp8 else "int8")
    side = {}
    if rank == 0 and not args.no_context:
        # the quantizer on its own rotation of inputs and outputs (> 3x L2 of its
        # bytes; the layer's buffer sets hold too few quantizer bytes for that)
        nq = max(2, int(np.ceil(3 * L2_BYTES / quant_bytes)))
        qsets = [(sets[0]["x"] if i == 0 else torch.roll(sets[0]["x"], shifts=i, dims=0).contiguous(),
                  torch.empty((M, K), dtype=code_dtype, device=dev),
                  torch.empty((M,), dtype=torch.float32, device=dev)) for i in range(nq)]

        def step_quant_rotating(i):
            x, xq, sa = qsets[i % nq]
            quantize_act(x, xq=xq, scale_a=sa, stream=stream)

        side["quant_ms"] = time_graph(step_quant_rotating, stream, dev, nq * max(1, 24 // nq), max(3, 300 // G))
        side["quant_rotation_mb"] = round(nq * quant_bytes / 2 ** 20, 1)
        del qsets
        if fp8 or args.no_per_config:
            # int8 runs time every entry point of every configuration in per_config
            side["gemm_ms"] = graph_ms(step_gemm, max(3, 300 // G))
            side["linear_ms"] = graph_ms(step_linear, max(3, 300 // G))
            if not fp8:
                side["fused_ms"] = graph_ms(step_fused, max(3, 300 // G))
        # the floor for the quantizer's byte count: a plain device copy moving
        # the same bytes (half read, half written), same harness, same rotation
        # (its own rotation, combined footprint > 3x L2, so that it is HBM traffic)
        half = quant_bytes // 2 // 16 * 16
        ncopy = max(2, int(np.ceil(3 * L2_BYTES / (2 * half))))
        copy_src = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(ncopy)]
        copy_dst = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(ncopy)]
        for t in copy_src:
            t.fill_(1)

        def step_copy(i):
            copy_dst[i % ncopy].copy_(copy_src[i % ncopy])

        side["copy_ms"] = graph_ms(step_copy, max(3, 300 // G))
        del copy_src, copy_dst
        side = {k: v for k, v in side.items() if v is not None}
    traffic = ncu_traffic(wl.name, "fp8" if fp8 else args.path)

    result = None
    if rank == 0:
        e2e = run_e2e(w8, wl, x_host, sets[0]["wq"], sw, bias, dev, stream, args) if args.e2e_steps else None
        with_table = not args.no_per_config and not fp8
        ctx = (context_baselines(wl, d, sets, sw, bias, dev, args, graph_ms)
               if not args.no_context and not with_table else
               {"see": "per_config (bf16_matmul, dequant_to_bf16_path, torch_int_mm_no_epilogue)"} if with_table
               else None)
        cpu = cpu_baseline(wl, fp8=fp8) if (world == 1 and not args.no_cpu_baseline) else None
        table = (per_config_table(w8, dev, stream, peaks, cpu=world == 1 and not args.no_cpu_baseline)
                 if with_table else None)
        cfg = wl_config(wl)
        cfg["format"] = "fp8 (OCP E4M3 codes, fp32 accumulation)" if fp8 else "int8 (int32 accumulation)"
        cfg["path"] = ("one fused kernel per step (w8a8_linear_fused)" if args.path == "fused"
                       else f"{linear.__name__} per step: quantizer kernel, then the GEMM kernel as its "
                            "programmatic dependent")
        cfg["timing"] = (f"CUDA graphs of {G} steps replayed, the last {G_inst} steps an instrumented graph "
                         f"(events around each GEMM); events around the whole timed region "
                         f"({elapsed_ms:.1f} ms)")
        cfg["parallelism"] = f"dp{world} (independent token batches, replicated weight)"
        cfg["gemm_config"] = w8.w8a8_select_config(M, N, K)
        cfg["buffer_sets"] = nsets
        cfg["footprint_mb"] = round(nsets * set_bytes / 2 ** 20, 1)
        kname = ("gemm_w8a8_kernel, fused (quantize + GEMM + epilogue)" if args.path == "fused"
                 else "gemm_w8a8_kernel (GEMM + dequant/bias epilogue)")
        unit = "TFLOPS" if fp8 else "TOPS"
        result = {
            "metric": METRIC_FP8 if fp8 else METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3" if fp8 else "int8",
            "data": "synthetic (seeded; stands in for Ideogram 4.0 "
            "DiT activations and weights, which are not available)", "config": cfg,
            "roofline": dict({"bound": "tensor", "achieved": kernel_tops, "peak": roof_peak["peak"],
                              "unit": unit, "frac": kernel_tops / roof_peak["peak"],
                              "traffic": traffic["dram_bytes_per_launch"] if traffic else None,
                              "kernel": kname, "ms_per_launch": kernel_ms,
                              "timing": f"CUDA events around each of the last {G_inst} launches of this kernel "
                                        "inside the timed region (on the launching stream)"},
                             **roof_peak["detail"](kernel_tops)),
            ("pct_of_spec_fp8_4p5_pflops" if fp8 else "pct_of_spec_int8_4p5_pops"): 100 * kernel_tops / SPEC_INT8_POPS,
            "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
            "cpu_baseline": cpu, "context": ctx, "per_config": table,
        }
        if side:
            result["components"] = {
                "note": "after the timed region: graphs of back-to-back calls of one entry point"
                        + ("" if not with_table else "; the GEMM, linear and fused entry points of every "
                           "configuration, this one included, are in per_config"),
            }
            if "quant_ms" in side:
                qg = quant_bytes / (side["quant_ms"] * 1e-3) / 1e9
                result["components"]["quantizer"] = {"ms": side["quant_ms"], "gbs": qg,
                                                     "rotation_mb": side["quant_rotation_mb"],
                                                     "frac_of_measured_hbm": qg / peaks["hbm_gbs"],
                                                     "frac_of_8tbs": qg / 8000.0, "bytes": quant_bytes}
                if "copy_ms" in side:
                    cg = 2 * (quant_bytes // 2 // 16 * 16) / (side["copy_ms"] * 1e-3) / 1e9
                    result["components"]["quantizer"]["copy_floor"] = {
                        "ms": side["copy_ms"], "gbs": cg, "frac_of_measured_hbm": cg / peaks["hbm_gbs"],
                        "what": "torch copy_ moving the quantizer's byte count (half read, half written), "
                                "graph of back-to-back calls over rotating buffers larger than 3x L2"}
            for key, name in (("gemm_ms", gemm.__name__), ("linear_ms", linear.__name__),
                              ("fused_ms", "w8a8_linear_fused")):
                if key in side:
                    tops = ops / (side[key] * 1e-3) / 1e12
                    result["components"][name] = {"ms": side[key], "tops": tops,
                                                  "pct_of_spec_int8_4p5_pops": 100 * tops / SPEC_INT8_POPS}
        print(json.dumps(result), flush=True)


def run_e2e(w8, wl, x_host, wq, sw, bias, dev, stream, args) -> dict:
    """The public API with host buffers, every step: its input X copied in
    from pinned host memory, the linear layer, its output copied back to
    pinned host memory; timed on the device from the first copy in to the
    last copy out.  Steps are pipelined as a serving loop would run them:
    three streams (copy in, compute, copy out) and two buffer sets, so step
    i+1's copy in and step i-1's copy out overlap step i's compute (PCIe is
    full duplex); event dependencies keep every buffer's reuse safe."""
    M, N, K = wl.M, wl.N, wl.K
    fp8 = args.format == "fp8"
    linear = w8.w8a8_linear_fp8 if fp8 else w8.w8a8_linear
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    B = 2
    xh = [x_host.pin_memory() for _ in range(B)]
    oh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(B)]
    xd = [torch.empty((M, K), dtype=torch.bfloat16, device=dev) for _ in range(B)]
    od = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(B)]
    xq = torch.empty((M, K), dtype=torch.uint8 if fp8 else torch.int8, device=dev)
    sa = torch.empty((M,), dtype=torch.float32, device=dev)
    sync = torch.zeros((w8.w8a8_linear_sync_words(M),), dtype=torch.int32, device=dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    copied_in = [ev() for _ in range(B)]
    computed = [ev() for _ in range(B)]
    copied_out = [ev() for _ in range(B)]
    used = [False] * B

    def one(i):
        b = i % B
        if used[b]:
            s_in.wait_event(computed[b])        # xd[b] is free once step i-B's layer has read it
        with torch.cuda.stream(s_in):
            xd[b].copy_(xh[b], non_blocking=True)
        copied_in[b].record(s_in)
        stream.wait_event(copied_in[b])
        if used[b]:
            stream.wait_event(copied_out[b])    # od[b] is free once step i-B's result is copied out
        if args.path == "fused":
            w8.w8a8_linear_fused(xd[b], wq, sw, bias, out=od[b], ws_xq=xq, ws_scale_a=sa, ws_sync=sync,
                                 stream=stream)
        else:
            linear(xd[b], wq, sw, bias, out=od[b], ws_xq=xq, ws_scale_a=sa, stream=stream)
        computed[b].record(stream)
        s_out.wait_event(computed[b])
        with torch.cuda.stream(s_out):
            oh[b].copy_(od[b], non_blocking=True)
        copied_out[b].record(s_out)
        used[b] = True

    for i in range(3):
        one(i)
    torch.cuda.synchronize(dev)
    steps = args.e2e_steps
    a = torch.cuda.Event(enable_timing=True)
    b_ev = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    stream.wait_event(a)
    s_out.wait_event(a)
    for i in range(steps):
        one(i)
    s_in.wait_event(copied_out[(steps - 1) % B])
    b_ev.record(s_in)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b_ev) / steps
    return {"value": 2.0 * M * N * K / (ms * 1e-3) / 1e12, "unit": "TFLOPS" if fp8 else "TOPS", "ms_per_step": ms,
            "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "steps": steps,
            "pipeline": "copy in / compute / copy out on three streams, two buffer sets"}


def context_baselines(wl, d, sets, sw, bias, dev, args, graph_ms) -> dict:
    """Context on the same shape, timed like the layer itself (a CUDA graph
    of back-to-back calls cycling through the same rotating buffer sets, so
    operands come from HBM): torch bf16 matmul (+bias), the
    dequantize-to-bf16-then-bf16-GEMM path the paper replaces, and the
    library low-precision GEMMs (torch._int_mm: int8 -> int32 without an
    epilogue; torch._scaled_mm: E4M3 with row-wise scales and bias)."""
    M, N, K = wl.M, wl.N, wl.K
    nsets = len(sets)
    w_bf16 = torch.from_numpy(d["w"]).to(dev).to(torch.bfloat16)
    w_sets = [w_bf16] + [w_bf16.clone() for _ in range(nsets - 1)]
    fp8 = args.format == "fp8"
    acc32 = [torch.empty((M, N), dtype=torch.int32, device=dev) for _ in range(nsets)] if not fp8 else []

    def bf16_matmul(i):
        s = sets[i % nsets]
        torch.addmm(bias, s["x"], w_sets[i % nsets].t(), out=s["out"])

    def torch_int_mm_no_epilogue(i):
        s = sets[i % nsets]
        torch._int_mm(s["xq"], s["wq"].t(), out=acc32[i % nsets])

    def torch_scaled_mm_fp8_rowwise(i):
        s = sets[i % nsets]
        torch._scaled_mm(s["xq"].view(torch.float8_e4m3fn), s["wq"].view(torch.float8_e4m3fn).t(),
                         scale_a=s["sa"][:, None], scale_b=sw[None, :], bias=bias, out_dtype=torch.bfloat16,
                         out=s["out"])

    def dequant_to_bf16_path(i):
        # the production "INT8" forward: quantize, dequantize to bf16, bf16 GEMM
        s = sets[i % nsets]
        xf = s["x"].float()
        sa = xf.abs().amax(dim=1, keepdim=True) / 127.0
        xq = torch.clamp(torch.round(xf / torch.where(sa > 0, sa, torch.ones_like(sa))), -127, 127)
        xd = (xq * sa).to(torch.bfloat16)
        wd = (s["wq"].float() * sw[:, None]).to(torch.bfloat16)
        torch.addmm(bias, xd, wd.t(), out=s["out"])

    out = {"timing": "CUDA graph of back-to-back calls over the rotating buffer sets (as the layer)"}
    cands = [bf16_matmul] + ([torch_scaled_mm_fp8_rowwise] if fp8 else [dequant_to_bf16_path,
                                                                        torch_int_mm_no_epilogue])
    for fn in cands:
        try:
            for i in range(3):
                fn(i)
            torch.cuda.synchronize(dev)
        except (RuntimeError, TypeError) as exc:  # not supported by this torch / device
            out[fn.__name__] = {"unavailable": str(exc).splitlines()[0][:200]}
            continue
        ms = graph_ms(fn, 10)
        if ms is None:
            out[fn.__name__] = {"unavailable": "could not be captured in a CUDA graph"}
            continue
        out[fn.__name__] = {"ms": ms, "tops": 2.0 * M * N * K / (ms * 1e-3) / 1e12}
    del w_sets, w_bf16, acc32
    return out


# ------------------------------------------------------ per-config table

# Every linear-layer configuration of the DiT workloads (QKV at 768px; the
# 1024px MLP up- and long-K down-projection; the four layers of the full-block
# sweep at batch 2, 1024px + 512 text tokens), each measured on its own in the
# same run as the headline line.
PER_CONFIG = ["qkv_768", "mlp_up_1024", "mlp_down_1024", "sweep_qkv", "sweep_out", "sweep_up", "sweep_down"]


def time_graph(fn, stream, dev, n: int, reps: int) -> float | None:
    """Mean ms per call of fn(i): a CUDA graph of n back-to-back calls
    (i = 0..n-1), replayed reps times between CUDA events on `stream`."""
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            for i in range(n):
                fn(i)
    except RuntimeError as exc:
        print(f"[bench] could not capture {getattr(fn, '__name__', fn)}: {exc}", file=sys.stderr)
        torch.cuda.synchronize(dev)
        return None
    g.replay()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_ev.record(stream)
    for _ in range(reps):
        g.replay()
    b_ev.record(stream)
    torch.cuda.synchronize(dev)
    return a_ev.elapsed_time(b_ev) / (reps * n)


def measure_config(w8, wl, dev, stream, peaks: dict, cpu: bool) -> dict:
    """One configuration, every entry point timed the same way: CUDA graphs
    of back-to-back calls cycling through buffer sets whose combined size is
    more than 3x L2, so operands come from HBM.  The seeded inputs of the
    workload; int8-given workloads (long-K MLP down) have no quantizer."""
    M, N, K = wl.M, wl.N, wl.K
    d = workloads.make(wl)
    linear_kind = wl.kind == "linear"
    bias = torch.from_numpy(d["bias"].view(np.int16)).view(torch.bfloat16).to(dev)
    if linear_kind:
        wq0, sw = w8.w8a8_quantize_weight(torch.from_numpy(d["w"]).to(dev))
        x0 = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).to(dev)
        w_bf = torch.from_numpy(d["w"]).to(dev).to(torch.bfloat16)
        set_bytes = M * K * 2 + M * K + N * K + N * K * 2 + M * N * 2 + 4 * M
    else:
        wq0 = torch.from_numpy(d["wq"]).to(dev)
        sw = torch.from_numpy(d["scale_w"]).to(dev)
        xq0 = torch.from_numpy(d["xq"]).to(dev)
        sa0 = torch.from_numpy(d["scale_a"]).to(dev)
        # the bf16 context runs on the dequantized operands
        x0 = (xq0.float() * sa0[:, None]).to(torch.bfloat16)
        w_bf = (wq0.float() * sw[:, None]).to(torch.bfloat16)
        set_bytes = M * K * 2 + M * K + N * K + N * K * 2 + M * N * 2 + 4 * M
    nsets = max(2, int(np.ceil(3 * L2_BYTES / set_bytes)))
    sets = []
    for i in range(nsets):
        s = {"x": x0 if i == 0 else torch.roll(x0, shifts=i, dims=0).contiguous(),
             "wq": wq0 if i == 0 else wq0.clone(), "w_bf": w_bf if i == 0 else w_bf.clone(),
             "out": torch.empty((M, N), dtype=torch.bfloat16, device=dev)}
        if linear_kind:
            s["xq"] = torch.empty((M, K), dtype=torch.int8, device=dev)
            s["sa"] = torch.empty((M,), dtype=torch.float32, device=dev)
            w8.w8a8_quantize_act(s["x"], xq=s["xq"], scale_a=s["sa"], stream=stream)
        else:
            s["xq"] = xq0 if i == 0 else torch.roll(xq0, shifts=i, dims=0).contiguous()
            s["sa"] = sa0 if i == 0 else torch.roll(sa0, shifts=i, dims=0).contiguous()
        sets.append(s)
    torch.cuda.synchronize(dev)

    def gemm(i):
        s = sets[i % nsets]
        w8.w8a8_gemm(s["xq"], s["wq"], s["sa"], sw, bias, out=s["out"], stream=stream)

    def linear(i):
        s = sets[i % nsets]
        w8.w8a8_linear(s["x"], s["wq"], sw, bias, out=s["out"], ws_xq=s["xq"], ws_scale_a=s["sa"], stream=stream)

    # the quantizer alone moves far fewer bytes than the layer: its own
    # rotation of inputs and outputs, more than 3x L2 in all
    qbytes = 3 * M * K + 4 * M
    nq = max(2, int(np.ceil(3 * L2_BYTES / qbytes))) if linear_kind else 0
    qsets = [(x0 if i == 0 else torch.roll(x0, shifts=i, dims=0).contiguous(),
              torch.empty((M, K), dtype=torch.int8, device=dev), torch.empty((M,), dtype=torch.float32, device=dev))
             for i in range(nq)]

    def quant(i):
        x, xq, sa = qsets[i % nq]
        w8.w8a8_quantize_act(x, xq=xq, scale_a=sa, stream=stream)

    def bf16_matmul(i):
        s = sets[i % nsets]
        torch.addmm(bias, s["x"], s["w_bf"].t(), out=s["out"])

    sync = [torch.zeros((w8.w8a8_linear_sync_words(M),), dtype=torch.int32, device=dev) for _ in range(nsets)]

    def fused(i):
        s = sets[i % nsets]
        w8.w8a8_linear_fused(s["x"], s["wq"], sw, bias, out=s["out"], ws_xq=s["xq"], ws_scale_a=s["sa"],
                             ws_sync=sync[i % nsets], stream=stream)

    acc32 = [torch.empty((M, N), dtype=torch.int32, device=dev) for _ in range(2)]

    def torch_int_mm_no_epilogue(i):
        # the library int8 GEMM (cuBLAS through torch) with int32 output, no dequantization
        s = sets[i % nsets]
        torch._int_mm(s["xq"], s["wq"].t(), out=acc32[i % 2])

    def dequant_to_bf16_path(i):
        # the production "INT8" forward the paper replaces: quantize, dequantize to bf16, bf16 GEMM
        s = sets[i % nsets]
        xf = s["x"].float()
        sa = xf.abs().amax(dim=1, keepdim=True) / 127.0
        xq = torch.clamp(torch.round(xf / torch.where(sa > 0, sa, torch.ones_like(sa))), -127, 127)
        wd = (s["wq"].float() * sw[:, None]).to(torch.bfloat16)
        torch.addmm(bias, (xq * sa).to(torch.bfloat16), wd.t(), out=s["out"])

    n = nsets * max(1, 12 // nsets)
    ops = 2.0 * M * N * K
    res = {"workload": wl.name, "M": M, "N": N, "K": K, "buffer_sets": nsets,
           "footprint_mb": round(nsets * set_bytes / 2 ** 20, 1)}
    gms = time_graph(gemm, stream, dev, n, 5)
    res["gemm_us"] = 1e3 * gms
    res["gemm_tops"] = ops / (gms * 1e-3) / 1e12
    res["gemm_pct_of_spec_4p5"] = 100 * res["gemm_tops"] / SPEC_INT8_POPS
    res["gemm_frac_of_burst_peak"] = res["gemm_tops"] / (peaks["bf16_tflops"] * NOMINAL_INT8_OVER_BF16)
    res["gemm_config"] = w8.w8a8_select_config(M, N, K)
    if linear_kind:
        fms = time_graph(fused, stream, dev, n, 5)
        res["fused_us"] = None if fms is None else 1e3 * fms
        lms = time_graph(linear, stream, dev, n, 5)
        qms = time_graph(quant, stream, dev, nq * max(1, 24 // nq), 5)
        res["quant_rotation_mb"] = round(nq * qbytes / 2 ** 20, 1)
        res["linear_us"] = 1e3 * lms
        res["linear_tops"] = ops / (lms * 1e-3) / 1e12
        res["linear_pct_of_spec_4p5"] = 100 * res["linear_tops"] / SPEC_INT8_POPS
        res["quant_us"] = 1e3 * qms
        res["quant_gbs"] = qbytes / (qms * 1e-3) / 1e9
        res["quant_frac_of_measured_hbm"] = res["quant_gbs"] / peaks["hbm_gbs"]
        res["quant_frac_of_8tbs"] = res["quant_gbs"] / 8000.0
    for fn in (bf16_matmul, dequant_to_bf16_path, torch_int_mm_no_epilogue):
        try:
            fn(0)
            torch.cuda.synchronize(dev)
        except (RuntimeError, TypeError) as exc:  # not supported by this torch / device
            res[fn.__name__ + "_us"] = {"unavailable": str(exc).splitlines()[0][:160]}
            continue
        ms = time_graph(fn, stream, dev, n, 3)
        res[fn.__name__ + "_us"] = None if ms is None else 1e3 * ms
    # The paper's accuracy metric on this configuration: the output of one
    # fresh call on the first buffer set against the float64 product on 64
    # sampled rows (of the unquantized operands for bf16 inputs; of the
    # dequantized codes where int8 codes are given), and NaNs in the whole
    # output.
    s0 = sets[0]
    (linear if linear_kind else gemm)(0)
    torch.cuda.synchronize(dev)
    rows = torch.linspace(0, M - 1, min(64, M), device=dev).round().long()
    b64 = bias.double()
    if linear_kind:
        ref = s0["x"][rows].double() @ torch.from_numpy(d["w"]).to(dev).double().t() + b64
    else:
        ref = (s0["xq"][rows].double() * s0["sa"][rows, None].double()) @ (
            s0["wq"].double() * sw[:, None].double()).t() + b64
    y = s0["out"][rows].double()
    res["accuracy"] = {"cosine_vs_fp64": float((y * ref).sum() / (y.norm() * ref.norm())),
                       "max_rel_err_vs_fp64": float(((y - ref).abs().max() / ref.abs().max())),
                       "nan_outputs": int(torch.isnan(s0["out"]).sum()),
                       "against": "unquantized operands" if linear_kind else "dequantized int8 codes",
                       "rows": int(rows.numel())}
    if cpu:
        work = OracleWork(wl, pool_rows=256)
        rows, cols = size_sample(work, 1.5)
        dt = work.sample(rows, cols)
        res["oracle"] = {"tops": 2.0 * rows * cols * K / dt / 1e12, "cores": work.threads,
                         "sample": f"{rows} tokens x {cols} channels, {dt:.2f} s",
                         "full_layer_s_extrapolated": dt * (M * N) / (rows * cols)}
    del sets, qsets, x0, w_bf, wq0, acc32, sync
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return res


def per_config_table(w8, dev, stream, peaks: dict, cpu: bool) -> dict:
    sampler = ClockSampler(dev.index)
    rows = [measure_config(w8, workloads.WORKLOADS[name], dev, stream, peaks, cpu) for name in PER_CONFIG]
    return {"note": "after the timed region, each configuration on its own: CUDA graphs of back-to-back calls "
                    "over rotating buffer sets (> 3x L2); gemm = w8a8_gemm (quantized operands given), linear = "
                    "w8a8_linear (quantizer + GEMM), fused = w8a8_linear_fused (one kernel), quant = "
                    "w8a8_quantize_act (its own rotation); bf16_matmul = torch.addmm; dequant_to_bf16_path = "
                    "quantize, dequantize to bf16, bf16 GEMM (the path the paper replaces); "
                    "torch_int_mm_no_epilogue = the library int8 GEMM, int32 out; oracle = the CPU oracle on a "
                    "row x column sample of the whole layer",
            "clocks": sampler.stop(), "configs": rows}


# ------------------------------------------------------- DiT block chain


def oracle_block_sample(blk, rows: int, d: dict, wq: dict) -> float:
    """Wall time of the oracle running `rows` tokens through every layer of the block."""
    import oracle
    sl = slice(0, rows)
    src = {"x": d["x"][sl], "a": d["a"][sl]}
    t0 = time.perf_counter()
    for l in blk.layers:
        x = oracle.gelu(src[l.source]) if l.act == "gelu" else src[l.source]
        out, _, _, _ = oracle.linear(x, wq[l.name][0], wq[l.name][1], d["bias_" + l.name])
        src[l.name] = out
    return time.perf_counter() - t0


def block_oracle_setup(blk, pool_rows: int = 256):
    import oracle
    d = blk.inputs(rows=slice(0, pool_rows))
    wq = {l.name: oracle.quantize_weight(d["w_" + l.name]) for l in blk.layers}
    return d, wq, oracle.default_threads()


def block_cpu_baseline(blk, budget_s: float = 12.0) -> dict:
    d, wq, cores = block_oracle_setup(blk)
    t1 = max(oracle_block_sample(blk, 2, d, wq) / 2, 1e-6)
    rows = int(max(1, min(256, budget_s / t1)))
    dt = oracle_block_sample(blk, rows, d, wq)
    ops = blk.ops / blk.M * rows
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle",
            "sample": f"{rows} of {blk.M} tokens through all {len(blk.layers)} layers of {blk.name} "
                      f"(quantize + exact GEMM + epilogue per layer), {dt:.2f} s", "seconds": dt}


def run_reference_block(args, blk) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    d, wq, cores = block_oracle_setup(blk)
    budget = 120.0 / max(1, args.steps + args.warmup)
    t1 = max(oracle_block_sample(blk, 2, d, wq) / 2, 1e-6)
    rows = int(max(1, min(256, budget / t1)))
    for _ in range(args.warmup):
        oracle_block_sample(blk, rows, d, wq)
    total = sum(oracle_block_sample(blk, rows, d, wq) for _ in range(args.steps))
    value = blk.ops / blk.M * rows * args.steps / total / 1e12
    sample = f"{rows} of {blk.M} tokens through all layers of {blk.name} per step"
    print(json.dumps({"impl": "reference", "metric": METRIC_BLOCK, "value": value, "unit": "TOPS",
                      "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
                      "vs_baseline": None, "dtype": "int64", "data": "synthetic", "config": block_config(blk),
                      "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                                       "sample": sample},
                      "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                      "gpu_launches": 0}), flush=True)


def block_e2e(args, blk, w8, L, host, dev, stream) -> dict:
    """The block through the chain API with host buffers, every step: the
    two block inputs copied in from pinned host memory, one chain launch,
    the QKV and MLP-down outputs copied back.  Pipelined like run_e2e: three
    streams, two chains recorded over two sets of input/output buffers (the
    weights, workspaces and the intermediate activations are shared; the
    compute stream runs the chains one after the other)."""
    first, last = blk.layers[0].name, blk.layers[-1].name
    B = 2
    ins, outs, chains = [], [], []
    for b in range(B):
        src = {k: torch.empty_like(L[blk.layers[0].name]["x"]) if k == "x" else torch.empty(
            (blk.M, 3072), dtype=torch.bfloat16, device=dev) for k in ("x", "a")}
        layers = []
        for l in blk.layers:
            t = L[l.name]
            out = torch.empty_like(t["out"]) if l.name in (first, last) else t["out"]
            x = src[l.source] if l.source in src else layers[[m.name for m in blk.layers].index(l.source)]["out"]
            layers.append(w8.linear_layer(x, t["wq"], t["scale_w"], t["bias"], out=out, ws_xq=t["ws_xq"],
                                          ws_scale_a=t["ws_scale_a"], input_act=t["input_act"]))
        ins.append(src)
        outs.append({first: layers[0]["out"], last: layers[-1]["out"]})
        chains.append(w8.w8a8_chain_create(layers))
    pin = [{k: host[k].pin_memory() for k in host} for _ in range(B)]
    ph = [{n: torch.empty(tuple(outs[0][n].shape), dtype=torch.bfloat16).pin_memory() for n in (first, last)}
          for _ in range(B)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    copied_in = [torch.cuda.Event() for _ in range(B)]
    computed = [torch.cuda.Event() for _ in range(B)]
    copied_out = [torch.cuda.Event() for _ in range(B)]
    used = [False] * B

    def one(i):
        b = i % B
        if used[b]:
            s_in.wait_event(computed[b])
        with torch.cuda.stream(s_in):
            for k in pin[b]:
                ins[b][k].copy_(pin[b][k], non_blocking=True)
        copied_in[b].record(s_in)
        stream.wait_event(copied_in[b])
        if used[b]:
            stream.wait_event(copied_out[b])
        chains[b].launch(stream)
        computed[b].record(stream)
        s_out.wait_event(computed[b])
        with torch.cuda.stream(s_out):
            for n in ph[b]:
                ph[b][n].copy_(outs[b][n], non_blocking=True)
        copied_out[b].record(s_out)
        used[b] = True

    for i in range(3):
        one(i)
    torch.cuda.synchronize(dev)
    steps = args.e2e_steps
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_ev.record(s_in)
    stream.wait_event(a_ev)
    s_out.wait_event(a_ev)
    for i in range(steps):
        one(i)
    s_in.wait_event(copied_out[(steps - 1) % B])
    b_ev.record(s_in)
    torch.cuda.synchronize(dev)
    for c in chains:
        c.close()
    ems = a_ev.elapsed_time(b_ev) / steps
    return {"value": blk.ops / (ems * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": ems,
            "h2d_bytes_per_step": sum(int(pin[0][k].numel()) * 2 for k in pin[0]),
            "d2h_bytes_per_step": sum(int(ph[0][n].numel()) * 2 for n in ph[0]), "steps": steps,
            "path": "w8a8_chain_launch with the block inputs copied in and the QKV and MLP-down outputs copied "
                    "out every step",
            "pipeline": "copy in / compute / copy out on three streams, two chains over two buffer sets"}


def block_config(blk) -> dict:
    return {"workload": f"{blk.name}: {blk.note}", "M": blk.M,
            "layers": [{"name": l.name, "N": l.N, "K": l.K, "input": l.source + (" (GELU)" if l.act else "")}
                       for l in blk.layers],
            "l2": "no rotation needed: one step moves ~0.9 GB, > 7x L2"}


def run_block(args, blk) -> None:
    import w8a8_int8_gemm_b200 as w8

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        _run_block_on(args, blk, w8, rank, world, local, dev, stream)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def _run_block_on(args, blk, w8, rank, world, local, dev, stream) -> None:
    M = blk.M
    d = blk.inputs(rows=rank_token_rows(M, rank))
    host = {k: torch.from_numpy(d[k].view(np.int16)).view(torch.bfloat16) for k in ("x", "a")}
    src = {k: host[k].to(dev) for k in host}
    L, wbf16 = {}, {}
    for l in blk.layers:
        w32 = torch.from_numpy(d["w_" + l.name]).to(dev)
        wq, sw = w8.w8a8_quantize_weight(w32)
        wbf16[l.name] = w32.to(torch.bfloat16)
        del w32
        bias = torch.from_numpy(d["bias_" + l.name].view(np.int16)).view(torch.bfloat16).to(dev)
        L[l.name] = w8.linear_layer(src[l.source], wq, sw, bias,
                                    input_act=w8.ACT_GELU if l.act == "gelu" else w8.ACT_NONE)
        src[l.name] = L[l.name]["out"]
    chain = w8.w8a8_chain_create([L[l.name] for l in blk.layers])
    for _ in range(args.warmup):
        chain.launch(stream)
    torch.cuda.synchronize(dev)
    if w8.w8a8_read_device_error() != 0:
        raise SystemExit("a kernel wait timed out during warm-up")

    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            for i in range(n):
                fn(i)
        return g

    # The last R steps of the timed region replay an instrumented graph of
    # the block with CUDA events around every GEMM launch (the GEMMs then
    # launch without the programmatic overlap the events would break).
    R = 3
    inst_ev = [[(torch.cuda.Event(enable_timing=True, external=True),
                 torch.cuda.Event(enable_timing=True, external=True)) for _ in blk.layers] for _ in range(R)]

    def quantize(t):
        q = w8.w8a8_quantize_act_gelu if t["input_act"] == w8.ACT_GELU else w8.w8a8_quantize_act
        q(t["x"], xq=t["ws_xq"], scale_a=t["ws_scale_a"], stream=stream)

    def linear(t):
        f = w8.w8a8_linear_gelu if t["input_act"] == w8.ACT_GELU else w8.w8a8_linear
        f(t["x"], t["wq"], t["scale_w"], t["bias"], out=t["out"], ws_xq=t["ws_xq"], ws_scale_a=t["ws_scale_a"],
          stream=stream)

    def step_inst(i):
        for j, l in enumerate(blk.layers):
            t = L[l.name]
            quantize(t)
            inst_ev[i][j][0].record(stream)
            w8.w8a8_gemm(t["ws_xq"], t["wq"], t["ws_scale_a"], t["scale_w"], t["bias"], out=t["out"], stream=stream)
            inst_ev[i][j][1].record(stream)

    g_inst = capture(step_inst, R)
    g_inst.replay()
    torch.cuda.synchronize(dev)
    steps = max(args.steps, R + 1)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    start.record(stream)
    for _ in range(steps - R):
        chain.launch(stream)
    g_inst.replay()
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dev)
    if w8.w8a8_read_device_error() != 0:
        raise SystemExit("a kernel wait timed out in the timed region")
    ms_step = elapsed_ms / steps
    value = blk.ops * world / (ms_step * 1e-3) / 1e12
    gemm_ms = {l.name: statistics.fmean(inst_ev[i][j][0].elapsed_time(inst_ev[i][j][1]) for i in range(R))
               for j, l in enumerate(blk.layers)}
    gemm_total = sum(gemm_ms.values())
    kernel_tops = blk.ops / (gemm_total * 1e-3) / 1e12

    peaks = measured_peaks()
    roof_peak = tensor_peak(peaks, elapsed_ms)
    if rank != 0:
        chain.close()
        return
    G = 10

    def graph_ms(fn, reps=5):
        g = capture(fn, G)
        g.replay()
        a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_ev.record(stream)
        for _ in range(reps):
            g.replay()
        b_ev.record(stream)
        torch.cuda.synchronize(dev)
        return a_ev.elapsed_time(b_ev) / (reps * G)

    comps = {"note": "after the timed region, one layer at a time: graphs of back-to-back calls; each quantizer "
                     "on its own rotation of inputs larger than 3x L2 in all; the linear layers' operands and "
                     "outputs are larger than L2"}
    def quantize_rotating_ms(t, K):
        """The layer's quantizer on its own rotation of inputs and outputs, more
        than 3x L2 in all (one input of 85 MB would stay in L2)."""
        nq = max(1, int(np.ceil(3 * L2_BYTES / (3 * M * K + 4 * M))))
        qs = [(t["x"] if i == 0 else torch.roll(t["x"], shifts=i, dims=0).contiguous(), torch.empty_like(t["ws_xq"]),
               torch.empty_like(t["ws_scale_a"])) for i in range(nq)]
        q = w8.w8a8_quantize_act_gelu if t["input_act"] == w8.ACT_GELU else w8.w8a8_quantize_act

        def one(i):
            x, xq, sa = qs[i % nq]
            q(x, xq=xq, scale_a=sa, stream=stream)

        ms = time_graph(one, stream, dev, nq * max(1, 10 // nq), 5)
        del qs
        return ms, nq

    for l in blk.layers:
        t = L[l.name]
        qms, nq = quantize_rotating_ms(t, l.K)
        lms = graph_ms(lambda i, t=t: linear(t))
        qbytes = 3 * M * l.K + 4 * M
        ops = 2.0 * M * l.N * l.K
        comps[l.name] = {"N": l.N, "K": l.K, "input_act": l.act or "none", "quantizer_rotation": nq,
                         "gemm_ms_live": gemm_ms[l.name],
                         "gemm_tops_live": ops / (gemm_ms[l.name] * 1e-3) / 1e12,
                         "linear_ms": lms, "quantizer_ms": qms, "quantizer_gbs": qbytes / (qms * 1e-3) / 1e9,
                         "quantizer_frac_of_measured_hbm": qbytes / (qms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "gemm_config": w8.w8a8_select_config(M, l.N, l.K)}
        if l.act == "gelu":
            # the same input unfused: a bf16 GELU kernel writes G, the quantizer reads it back
            g = torch.empty_like(t["x"])
            gms = graph_ms(lambda i, t=t, g=g: w8.w8a8_gelu(t["x"], g, stream=stream))
            uqms = graph_ms(lambda i, t=t, g=g: w8.w8a8_quantize_act(g, xq=t["ws_xq"], scale_a=t["ws_scale_a"],
                                                                        stream=stream))
            comps[l.name]["unfused_gelu_ms"] = gms
            comps[l.name]["unfused_quantizer_ms"] = uqms
            comps[l.name]["fused_saves_ms"] = gms + uqms - qms
            del g
    ctx = None
    if not args.no_context:
        bsrc = {"x": src["x"], "a": src["a"]}
        bout = {l.name: torch.empty((M, l.N), dtype=torch.bfloat16, device=dev) for l in blk.layers}

        def bf16_block(i):
            for l in blk.layers:
                xin = bsrc[l.source] if l.source in bsrc else bout[l.source]
                if l.act == "gelu":
                    xin = torch.nn.functional.gelu(xin, approximate="tanh")
                torch.addmm(L[l.name]["bias"], xin, wbf16[l.name].t(), out=bout[l.name])

        for i in range(2):  # library handles are created outside graph capture
            bf16_block(i)
        torch.cuda.synchronize(dev)
        bms = graph_ms(bf16_block, 3)
        ctx = {"timing": "CUDA graph of back-to-back blocks", "bf16_matmul_chain": {"ms": bms,
               "tops": blk.ops / (bms * 1e-3) / 1e12}}
        del bout
    e2e = None
    if args.e2e_steps:
        e2e = block_e2e(args, blk, w8, L, host, dev, stream)
    cpu = block_cpu_baseline(blk) if (world == 1 and not args.no_cpu_baseline) else None
    block_traffic = ncu_traffic(blk.name, "block")
    cfg = block_config(blk)
    cfg["path"] = "w8a8_chain_launch per step: one CUDA graph of 4 x (quantizer + GEMM)"
    cfg["parallelism"] = f"dp{world} (independent token batches, replicated weights)"
    cfg["timing"] = (f"{steps} steps between CUDA events; the last {R} replay an instrumented graph with events "
                     "around each GEMM")
    result = {
        "metric": METRIC_BLOCK, "value": value, "unit": "TOPS", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded; stands in for Ideogram 4.0 "
        "DiT activations and weights, which are not available)", "config": cfg,
        "roofline": dict({"bound": "tensor", "achieved": kernel_tops, "peak": roof_peak["peak"], "unit": "TOPS",
                          "frac": kernel_tops / roof_peak["peak"],
                          "traffic": block_traffic["dram_bytes_per_launch"] if block_traffic else None,
                          "kernel": "gemm_w8a8_kernel over the block's four shapes (sum of their ops / sum of "
                                    "their live launch times; traffic: mean DRAM bytes of the four launches)",
                          "ms_per_launch": gemm_total / len(blk.layers),
                          "timing": f"CUDA events around each GEMM launch of the last {R} steps of the timed "
                                    "region"}, **roof_peak["detail"](kernel_tops)),
        "components": comps, "e2e": e2e, "gpu_launches": 2 * len(blk.layers) * steps, "clocks": clocks,
        "cpu_baseline": cpu, "context": ctx,
    }
    print(json.dumps(result), flush=True)
    chain.close()


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=12000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=workloads.HEADLINE,
                    choices=sorted(workloads.WORKLOADS) + sorted(workloads.BLOCKS),
                    help="a linear-layer workload, or a DiT block (its linears as one CUDA graph)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--path", default="two-kernel", choices=["fused", "two-kernel"],
                    help="w8a8_linear (quantizer + GEMM, default) or the one-kernel w8a8_linear_fused")
    ap.add_argument("--format", default="int8", choices=["int8", "fp8"],
                    help="int8 W8A8 (default) or its FP8 (E4M3) variant")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-context", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the table of every DiT configuration measured after the headline")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload in workloads.BLOCKS:
        blk = workloads.BLOCKS[args.workload]
        if args.format != "int8" or args.path != "two-kernel":
            ap.error("the block chain runs the int8 two-kernel layers")
        if args.impl == "reference":
            run_reference_block(args, blk)
        else:
            run_block(args, blk)
        return 0
    wl = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_native(args, wl)
    return 0


if __name__ == "__main__":
    sys.exit(main())
