"""Benchmark of the MX block-quantized linear layer on B200.

A step is one pass of the hot path over one batch: the dynamic activation quantizer
followed by the block-scaled tcgen05 GEMM (mxq_linear), on the W4A4 FFN-up linear of a
Wan2.2-A14B-shaped DiT block at 720p / 81 frames (M = 75600 tokens, K = 5120, N = 13824;
Student-t activations with 1% outlier channels, N(0, 0.02^2) weights, random-init,
synthetic), the shape the 60 %-of-FP4 target is stated for.  The MXFP4 weight is quantized
once, before timing (a load-time step).  Beside the headline number the JSON line carries:
  step_ms       median / min / p90 of the timed steps (events around every step);
  roofline      the dominant kernel (the GEMM) against the tensor-core peak: its average
                launch inside the timed region (events between the step's two launches,
                on their stream), as a fraction of the measured-derived peak and of the
                nominal 9 PFLOP/s;
  parts         the quantizer (GB/s against HBM) and the GEMM separately, inside the
                timed region and, beside that, each alone over 50 back-to-back launches;
  ffn_up_480p_w4a4  the same linear at 480p / 81 frames (M = 32760);
  w4a8          the W4A8 FFN-down linear at 720p (quantize to E4M3 + mxf8f6f4 GEMM),
                its quantize-dequantize emulation (QDQ) path, and the same linear with
                static per-tensor E4M3 activations;
  transform_720p  the transform_on quantizer (SmoothQuant scales + block Hadamard) and
                linear on the headline workload;
  lowrank_720p  the headline linear with an SVDQuant bf16 rank-64 / 128 branch in the same
                accumulator;
  ffn_720p      the block's FFN with its hidden activation kept MX-quantized (the
                FFN-up GEMM's epilogue applies GELU and quantizes), FFN-down W4A4 or W4A8;
  dit_block_720p  one DiT block's eight linears under the all-W4A4, all-W4A8 and mixed
                masks;
  expert_stack_480p  the two-expert stack of 40 blocks, MXFP4 weights resident, one
                expert's forward per timed unit;
  e2e           the same step through host buffers (pinned H2D of x, D2H of y every step),
                copies of neighbouring steps overlapped on separate streams; the serial
                form beside it;
  cpu_baseline  the CPU oracle on this machine's host cores: the linear on a bounded sample of
                rows and the quantizer on the whole activation, single-threaded and on all
                cores.

Multi-GPU: the layer has no exchange step (token rows are independent), so N GPUs
run N replicas, each on its own batch (weak scaling, no collective on the data path);
the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_FP4_TFLOPS = 9000.0   # dense FP4, nominal (the figure the roofline reporting names)
NOMINAL_HBM_GBS = 8000.0
FP4_OVER_BF16 = 4.0   # nominal dense ratio: 9 PFLOP/s FP4 vs 2.25 PFLOP/s bf16
FP8_OVER_BF16 = 2.0   # 4.5 PFLOP/s FP8


# DRAM traffic of one GEMM launch on a bench workload (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture of that launch).  A record describes only the
# kernel built from the sources it was taken on: when their hash differs the line reports
# traffic as null.
GEMM_SOURCES = ["fp8_mixed_precision_mxq_b200/csrc/gemm.cu", "fp8_mixed_precision_mxq_b200/csrc/ptx.cuh",
                "fp8_mixed_precision_mxq_b200/csrc/mxq_internal.h", "fp8_mixed_precision_mxq_b200/csrc/mx_elem.cuh"]
GEMM_TRAFFIC = {
    ("ffn_up_720p_w4a4", 75600): {
        "bytes": 662759936 + 2048216576,
        "sources_sha256": "675093c7b3b204cfe9b1b37c800248eaea482b08cddd63523ef23a2e233f80ae"},
}


def gemm_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gemm_traffic(workload: str, M: int):
    rec = GEMM_TRAFFIC.get((workload, M))
    if rec is None or rec["sources_sha256"] != gemm_sources_sha256():
        return None
    return rec["bytes"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.02)  # the timed region starts once sampling is live
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self):
        sm, smax, watts, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            try:
                watts.append(float(parts[2]))
            except ValueError:
                pass
            for name, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w": statistics.median(watts) if watts else None}


# ---------------------------------------------------------------------------- timing
def time_loop(fn, iters: int, stream) -> float:
    """Average milliseconds of fn() over iters runs, CUDA events on `stream`."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(iters):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / iters


def time_steps(fn, iters: int, stream):
    """(total ms, per-step ms list) of iters runs of fn(): one CUDA event before the first
    run, one after each, all on `stream`; the per-step times come from the same timed
    region as the total."""
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(iters + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(iters):
        fn()
        ev[i + 1].record(stream)
    ev[-1].synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(iters)]
    return ev[0].elapsed_time(ev[-1]), per


def time_steps_parts(parts, iters: int, stream):
    """iters steps, each the calls in `parts` in order, with a CUDA event on `stream` after
    every call.  Returns (total ms, per-step ms, per-part ms lists) from the one timed
    region."""
    n = len(parts)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(iters * n + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(iters):
        for j, fn in enumerate(parts):
            fn()
            ev[i * n + j + 1].record(stream)
    ev[-1].synchronize()
    per_step = [ev[i * n].elapsed_time(ev[(i + 1) * n]) for i in range(iters)]
    per_part = [[ev[i * n + j].elapsed_time(ev[i * n + j + 1]) for i in range(iters)] for j in range(n)]
    return ev[0].elapsed_time(ev[-1]), per_step, per_part


def step_stats(per):
    """median / min / p90 / mean of per-step milliseconds."""
    v = sorted(per)
    p90 = v[min(len(v) - 1, int(round(0.9 * (len(v) - 1))))]
    return {"median": round(statistics.median(v), 4), "min": round(v[0], 4), "p90": round(p90, 4),
            "mean": round(sum(v) / len(v), 4), "n": len(v)}


def time_kernel(fn, stream, min_iters: int = 50, min_ms: float = 0.0, idle_s: float = 0.0):
    """A kernel timed alone on its stream: min_iters launches, more if needed to fill min_ms
    of device time (a short probe sizes the loop), one event per launch, after idle_s
    seconds with the GPU idle (a preceding loop of GEMMs leaves the SM clock below its
    maximum for a while, which the partly issue-bound quantizers feel).  Returns the mean
    launch time (ms) and the per-launch statistics."""
    if idle_s > 0:
        torch.cuda.synchronize()
        time.sleep(idle_s)
    probe = time_loop(fn, 3, stream)
    iters = max(min_iters, int(min_ms / max(probe, 1e-3)) + 1)
    total, per = time_steps(fn, iters, stream)
    return total / iters, step_stats(per)


# seconds of idle GPU before each stand-alone quantizer loop that follows GEMM loops
QUANT_IDLE_S = 1.0


def quant_bytes(M, K, fmt):
    return 2 * M * K + (M * K if fmt == "e4m3" else M * K // 2) + M * K // 32


# ---------------------------------------------------------------------------- CPU oracle
def cpu_model() -> str:
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except (OSError, subprocess.SubprocessError):
        pass
    return "unknown"


_CPU_WEIGHTS = {}


def _cpu_weight(N, K, seed, nthreads):
    """The workload's weight quantized by the oracle, prepared once per process (load-time
    work, outside every timed sample)."""
    import numpy as np

    import oracle
    import synth
    key = (N, K, seed)
    if key not in _CPU_WEIGHTS:
        w = synth.weight(N, K, seed=seed)
        _CPU_WEIGHTS[key] = oracle.quantize(w.view(torch.int16).numpy().view(np.uint16), oracle.E2M1, nthreads)
    return _CPU_WEIGHTS[key]


def cpu_gemm_rate(M, N, K, fmt, seed, budget_s, nthreads):
    """The CPU oracle's quantize + fp64 linear on activation rows against a pre-quantized
    weight, for about budget_s seconds: (TFLOP/s, rows done, seconds)."""
    import numpy as np

    import oracle
    import synth
    f = oracle.E2M1 if fmt == "e2m1" else oracle.E4M3
    wc, ws = _cpu_weight(N, K, seed, nthreads)
    chunk = max(4, 4 * nthreads)
    rows_done, flops = 0, 0.0
    t0 = time.perf_counter()
    while True:
        x = synth.activation(chunk, K, "student_t" if fmt == "e2m1" else "gelu", seed=seed + rows_done,
                             outlier_frac=0.01, outlier_scale=50.0)
        xc, xs = oracle.quantize(x.view(torch.int16).numpy().view(np.uint16), f, nthreads)
        oracle.linear(xc, xs, f, K, wc, ws, nthreads=nthreads)
        flops += 2.0 * chunk * N * K
        rows_done += chunk
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, rows_done, dt


def cpu_quantize_rate(x_bits, fmt, nthreads):
    """The CPU oracle's quantizer on the whole activation tensor: (GB/s, seconds), bytes
    counted as the GPU quantizer's (bf16 in, codes and scales out)."""
    import oracle
    f = oracle.E2M1 if fmt == "e2m1" else oracle.E4M3
    M, K = x_bits.shape
    t0 = time.perf_counter()
    oracle.quantize(x_bits, f, nthreads)
    dt = time.perf_counter() - t0
    return quant_bytes(M, K, fmt) / dt / 1e9, dt


def cpu_baseline(M, N, K, fmt, seed, budget_s=6.0, x_bits=None):
    """The CPU oracle as it stands, on the host's CPU cores: the linear (quantize + fp64 GEMM)
    on a bounded sample of activation rows, single-threaded and on all cores (about budget_s
    seconds each), and, when the activation's bits are given, the quantizer on the whole
    tensor, single-threaded and on all cores.  `value` is the all-core linear rate."""
    import oracle
    cores = oracle.default_threads()
    g1, r1, t1 = cpu_gemm_rate(M, N, K, fmt, seed, budget_s, 1)
    ga, ra, ta = cpu_gemm_rate(M, N, K, fmt, seed, budget_s, cores)
    out = {"value": ga, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
           "sample": "%d of %d activation rows of the %dx%dx%d %s linear (quantize + fp64 GEMM on the "
                     "dequantized operands; weight quantized beforehand), %.1f s on %d threads; single thread: "
                     "%d rows in %.1f s" % (ra, M, M, N, K, fmt, ta, cores, r1, t1),
           "linear": {"TFLOP/s_all_cores": ga, "TFLOP/s_1_thread": g1,
                      "full_M_extrapolated_s_all_cores": round(2.0 * M * N * K / (ga * 1e12), 1)}}
    if x_bits is not None:
        q1, s1 = cpu_quantize_rate(x_bits, fmt, 1)
        qa, sa = cpu_quantize_rate(x_bits, fmt, cores)
        out["quantize"] = {"GB/s_all_cores": round(qa, 4), "GB/s_1_thread": round(q1, 4),
                           "s_all_cores": round(sa, 2), "s_1_thread": round(s1, 2),
                           "tensor": "the whole %dx%d activation (%.0f MB of bf16)" % (
                               x_bits.shape[0], x_bits.shape[1], x_bits.size * 2 / 1e6)}
    return out


# ---------------------------------------------------------------------------- main arms
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it); one all-reduce, on the
    process group's device (cuda under nccl, cpu under gloo)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def replica_seed(seed: int, rank: int) -> int:
    """Seed of a replica's activation batch: every rank quantizes its own tokens."""
    return seed + 1000 * rank


def job_tflops(flops_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput of `world` replicas that each did flops_per_rank in at most
    ms_max milliseconds."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def run_mxq(args):
    import synth
    from fp8_mixed_precision_mxq_b200 import ops

    world, rank, local = dist_setup()
    peaks, peak_src = load_peaks()
    wl_name = args.workload
    c = synth.WORKLOADS[wl_name]
    M, K, N, fmt = (args.M or c["M"]), c["K"], c["N"], c["fmt"]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    if args.only == "block":
        return profile_block(args, ops, synth, dev, stream)

    # inputs (per-rank seed offset: every replica gets its own batch)
    x = synth.activation(M, K, c["act"], seed=replica_seed(c["seed"], rank), device=dev,
                         outlier_frac=c.get("outlier_frac", 0.0), outlier_scale=c["outlier_scale"])
    w = synth.weight(N, K, seed=c["seed"], device=dev)
    b = synth.bias(N, seed=c["seed"], device=dev)
    qw = ops.quantize_weight(w, bias=b)
    ws = torch.empty(ops.workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    assert ops.poll_status() == 0

    # the timed step is mxq_linear's native path issued as its two launches, the quantizer
    # into the workspace and the GEMM on it, so that each kernel's time inside the timed
    # region can be read from events between them (the same kernels on the same buffers
    # as one mxq_linear call)
    xc = ws[: ops.codes_bytes(M, K, fmt)]
    xs_off = (ops.codes_bytes(M, K, fmt) + 255) // 256 * 256
    xs = ws[xs_off: xs_off + ops.sf_bytes(M, K)]

    def quant():
        ops.quantize_act(x, fmt, codes=xc, sf=xs)

    def gemm():
        ops.gemm(xc, xs, fmt, M, K, qw, out=y)

    def step():
        quant()
        gemm()

    if args.only:
        # profiling mode: only the named kernel, `steps` launches after the warm-up
        return profile_one(args, ops, x, qw, ws, y, M, N, K, fmt, stream)

    for _ in range(args.warmup):
        step()
    barrier(world)
    with ClockSampler(local) as clk:
        barrier(world)
        ms_total, per_step, (per_q, per_g) = time_steps_parts([quant, gemm], args.steps, stream)
        barrier(world)
    gemm_path = ops.last_path()
    # beside them: each kernel timed alone, 50 launches back to back (a long loop: the
    # GEMM runs into the 1 kW power cap there)
    q_alone, q_alone_stats = time_kernel(quant, stream)
    g_alone, g_alone_stats = time_kernel(gemm, stream)
    ms = max_over_ranks(ms_total / args.steps, world)
    status = ops.poll_status()
    if status != 0:
        raise RuntimeError("device status %d after the timed steps" % status)
    flops = 2.0 * M * N * K
    value = job_tflops(flops, ms, world)
    q_stats, g_stats = step_stats(per_q), step_stats(per_g)
    q_ms = max_over_ranks(sum(per_q) / len(per_q), world)   # average launch inside the timed region
    g_ms = max_over_ranks(sum(per_g) / len(per_g), world)
    q_alone, g_alone = max_over_ranks(q_alone, world), max_over_ranks(g_alone, world)
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    g_tflops = flops / (g_ms * 1e-3) / 1e12
    q_gbs = quant_bytes(M, K, fmt) / (q_ms * 1e-3) / 1e9

    result = {
        "metric": "W4A4 MX linear TFLOP/s (fused dynamic MXFP4 activation quantize + tcgen05 mxf4 GEMM)",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1 x e2m1 -> fp32 accumulate -> bf16", "data": "synthetic",
        "config": {"workload": "%s: Wan2.2-A14B FFN-up linear, M=%d K=%d N=%d, W4A4 (MXFP4 act + MXFP4 weight), "
                               "bias, bf16 out" % (wl_name, M, K, N),
                   "M": M, "K": K, "N": N, "act_fmt": fmt, "parallelism": "replicas%d" % world,
                   "l2": "inputs larger than L2 (x %.0f MB, y %.0f MB; L2 126 MB)" % (M * K * 2 / 1e6,
                                                                                       M * N * 2 / 1e6)},
        "step_ms": step_stats(per_step),
        "roofline": {"bound": "tensor", "kernel": "mx_gemm_kernel<mxf4>", "achieved": round(g_tflops, 1),
                     "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(g_tflops / fp4_peak, 4),
                     "peak_source": "%s bf16 burst %.1f TFLOP/s x %.0f (nominal FP4/bf16 dense ratio)" % (
                         peak_src, peaks["bf16_tflops"], FP4_OVER_BF16),
                     "frac_nominal": round(g_tflops / NOMINAL_FP4_TFLOPS, 4),
                     "nominal_peak": NOMINAL_FP4_TFLOPS,
                     # against the bf16 loop of seconds under the power cap (x the same ratio),
                     # the regime a long run of steps reaches; the clocks key says which it was
                     "frac_sustained": round(g_tflops / (sustained_tflops(peaks) * FP4_OVER_BF16), 4),
                     "ms": round(g_ms, 4), "launch_ms": g_stats, "traffic": gemm_traffic(wl_name, M),
                     "path": gemm_path},
        "parts": {
            "quantize": {"ms": round(q_ms, 4), "GB/s": round(q_gbs, 1), "peak_GB/s": peaks["hbm_gbs"],
                         "frac_hbm": round(q_gbs / peaks["hbm_gbs"], 4),
                         "frac_nominal_hbm": round(q_gbs / NOMINAL_HBM_GBS, 4),
                         "bytes": quant_bytes(M, K, fmt), "launch_ms": q_stats,
                         "alone_50": {"ms": round(q_alone, 4),
                                      "GB/s": round(quant_bytes(M, K, fmt) / (q_alone * 1e-3) / 1e9, 1),
                                      "launch_ms": q_alone_stats}},
            "gemm": {"ms": round(g_ms, 4), "TFLOP/s": round(g_tflops, 1),
                     "frac_fp4": round(g_tflops / fp4_peak, 4),
                     "alone_50": {"ms": round(g_alone, 4), "TFLOP/s": round(flops / (g_alone * 1e-3) / 1e12, 1),
                                  "frac_fp4": round(flops / (g_alone * 1e-3) / 1e12 / fp4_peak, 4),
                                  "launch_ms": g_alone_stats}},
        },
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }

    if args.extra_linear:
        result["ffn_up_480p_w4a4"] = bench_linear(args, ops, synth, "ffn_up_480p_w4a4", dev, stream, world, rank,
                                                  peaks)
    if args.w4a8:
        result["w4a8"] = bench_w4a8(args, ops, synth, dev, stream, world, rank, peaks)
    if args.transform:
        result["transform_720p"] = bench_transform(args, ops, synth, dev, stream, world, rank, peaks, x, w, b)
    if args.lowrank:
        result["lowrank_720p"] = bench_lowrank(args, ops, synth, dev, stream, world, rank, peaks, x, b)
    if args.ffn:
        result["ffn_720p"] = bench_ffn(args, ops, synth, dev, stream, world, rank, peaks)
    if args.block:
        result["dit_block_720p"] = bench_block(args, ops, synth, dev, stream, world, rank, peaks)
    if args.stack:
        result["expert_stack_480p"] = bench_stack(args, ops, synth, dev, stream, world, rank, peaks)

    # end to end: host buffers, H2D of x and D2H of y of every step inside the timed region
    if args.e2e:
        result["e2e"] = bench_e2e(args, ops, x, qw, fmt, ws, M, N, K, flops, world, dev)
    if rank == 0 and world == 1 and args.cpu_baseline:
        import numpy as np
        xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
        result["cpu_baseline"] = cpu_baseline(M, N, K, fmt, c["seed"], budget_s=args.cpu_seconds, x_bits=xb)
        del xb
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def bench_e2e(args, ops, x, qw, fmt, ws, M, N, K, flops, world, dev):
    """The step through the public API with host buffers: each step copies its input from
    pinned host memory, runs mxq_linear, and copies its result back to pinned host memory.
    Pipelined: step i's H2D copy, linear and D2H copy run on three streams with two device
    and host buffers per direction, so the H2D of step i+1 and the D2H of step i-1 overlap
    the linear of step i (the two copy directions use separate copy engines); events order
    every buffer reuse.  Timed from the first H2D to the last D2H with CUDA events.  The
    serial form (one stream, copies and linear back to back) is reported beside it."""
    xh = [x.cpu().pin_memory() for _ in range(2)]
    yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    yd = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            bb = i % 2
            if i >= 2:
                s_in.wait_event(ev_cmp[bb])  # the linear of step i-2 has read xd[bb]
            with torch.cuda.stream(s_in):
                xd[bb].copy_(xh[bb], non_blocking=True)
            ev_in[bb].record(s_in)
            s_cmp.wait_event(ev_in[bb])
            if i >= 2:
                s_cmp.wait_event(ev_out[bb])  # the D2H of step i-2 has read yd[bb]
            ops.linear(xd[bb], qw, fmt=fmt, workspace=ws, out=yd[bb], stream=s_cmp)
            ev_cmp[bb].record(s_cmp)
            s_out.wait_event(ev_cmp[bb])
            with torch.cuda.stream(s_out):
                yh[bb].copy_(yd[bb], non_blocking=True)
            ev_out[bb].record(s_out)

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    n = max(3, args.steps // 4)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    run(n)
    end.record(s_out)
    end.synchronize()
    p_ms = max_over_ranks(start.elapsed_time(end) / n, world)

    stream = torch.cuda.current_stream()

    def serial_step():
        xd[0].copy_(xh[0], non_blocking=True)
        ops.linear(xd[0], qw, fmt=fmt, workspace=ws, out=yd[0])
        yh[0].copy_(yd[0], non_blocking=True)

    for _ in range(2):
        serial_step()
    barrier(world)
    s_ms = max_over_ranks(time_loop(serial_step, n, stream), world)
    return {"value": round(job_tflops(flops, p_ms, world), 2), "unit": "TFLOP/s", "ms_per_step": round(p_ms, 3),
            "steps": n, "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
            "pipelined": True, "serial_ms_per_step": round(s_ms, 3),
            "serial_value": round(job_tflops(flops, s_ms, world), 2)}


def profile_one(args, ops, x, qw, ws, y, M, N, K, fmt, stream):
    xc = ws[: ops.codes_bytes(M, K, fmt)]
    off = (ops.codes_bytes(M, K, fmt) + 255) // 256 * 256
    xs = ws[off: off + ops.sf_bytes(M, K)]
    ops.quantize_act(x, fmt, codes=xc, sf=xs)
    if args.only == "gemm":
        fn = lambda: ops.gemm(xc, xs, fmt, M, K, qw, out=y)  # noqa: E731
    elif args.only == "gelu_quant":
        hc = torch.empty(ops.codes_bytes(M, N, "e2m1"), dtype=torch.uint8, device=x.device)
        hs = torch.empty(ops.sf_bytes(M, N), dtype=torch.uint8, device=x.device)
        fn = lambda: ops.gemm_gelu_quant(xc, xs, fmt, M, K, qw, out_fmt="e2m1", codes=hc, sf=hs)  # noqa: E731
    elif args.only == "transform":
        mul = torch.ones(K, dtype=torch.float32, device=x.device)
        fn = lambda: ops.quantize_act_transformed(x, fmt, args.rot_block, mul, codes=xc, sf=xs)  # noqa: E731
    elif args.only == "quantize_static":
        codes8 = torch.empty(ops.codes_bytes(M, K, "e4m3"), dtype=torch.uint8, device=x.device)
        scale = ops.absmax(x).item() / 448.0
        fn = lambda: ops.quantize_act_static(x, scale, codes=codes8, sf=xs)  # noqa: E731
    elif args.only == "gemm_bf16":
        xd = ops.dequantize(xc, xs, M, K, fmt)
        wd = ops.dequantize(qw.codes, qw.sf, N, K, "e2m1")
        fn = lambda: ops.gemm_bf16(xd, wd, qw.bias, out=y)  # noqa: E731
    elif args.only == "dequantize":
        xd = torch.empty((M, K), dtype=torch.bfloat16, device=x.device)
        fn = lambda: ops.dequantize(xc, xs, M, K, fmt, out=xd)  # noqa: E731
    elif args.only == "u_quantize":  # the low-rank branch's u (rank 64) with x's MX codes
        l1t = (torch.randn(64, K, device=x.device) * 0.02).to(torch.bfloat16)
        u = torch.empty((M, 64), dtype=torch.bfloat16, device=x.device)
        fn = lambda: ops.gemm_bf16_quant_a(x, l1t, fmt, out=u, codes=xc, sf=xs)  # noqa: E731
    else:
        fn = lambda: ops.quantize_act(x, fmt, codes=xc, sf=xs)  # noqa: E731
    for _ in range(args.warmup):
        fn()
    ms = time_loop(fn, args.steps, stream)
    status = ops.poll_status()
    print(json.dumps({"only": args.only, "workload": args.workload, "M": M, "N": N, "K": K, "fmt": fmt,
                      "rot_block": args.rot_block, "ms": round(ms, 4), "status": status, "path": ops.last_path()}))
    if status != 0:
        raise RuntimeError("device status %d" % status)


def bench_linear(args, ops, synth, wl_name, dev, stream, world, rank, peaks):
    """Another W4A4 linear workload beside the headline one (the FFN-up linear at 480p /
    81 frames, M = 32760): the whole step, then its GEMM and quantizer timed alone."""
    c = synth.WORKLOADS[wl_name]
    M, K, N = c["M"], c["K"], c["N"]
    x = synth.activation(M, K, c["act"], seed=replica_seed(c["seed"], rank), device=dev,
                         outlier_frac=c["outlier_frac"], outlier_scale=c["outlier_scale"])
    qw = ops.quantize_weight(synth.weight(N, K, seed=c["seed"], device=dev),
                             bias=synth.bias(N, seed=c["seed"], device=dev))
    ws = torch.empty(ops.workspace_bytes(M, N, K, "e2m1"), dtype=torch.uint8, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flops = 2.0 * M * N * K
    iters = max(3, args.steps // 4)
    for _ in range(2):
        ops.linear(x, qw, "e2m1", workspace=ws, out=y)
    ms = max_over_ranks(time_loop(lambda: ops.linear(x, qw, "e2m1", workspace=ws, out=y), iters, stream), world)
    xc = ws[: ops.codes_bytes(M, K, "e2m1")]
    off = (ops.codes_bytes(M, K, "e2m1") + 255) // 256 * 256
    xs = ws[off: off + ops.sf_bytes(M, K)]
    g_ms = max_over_ranks(time_loop(lambda: ops.gemm(xc, xs, "e2m1", M, K, qw, out=y), iters, stream), world)
    q_ms = max_over_ranks(time_kernel(lambda: ops.quantize_act(x, "e2m1", codes=xc, sf=xs), stream,
                                      idle_s=QUANT_IDLE_S)[0], world)
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    if ops.poll_status() != 0:
        raise RuntimeError("device status set during the %s measurement" % wl_name)
    q_gbs = quant_bytes(M, K, "e2m1") / (q_ms * 1e-3) / 1e9
    return {"workload": "%s: M=%d K=%d N=%d W4A4" % (wl_name, M, K, N),
            "linear": {"ms": round(ms, 4), "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1)},
            "gemm": {"ms": round(g_ms, 4), "TFLOP/s": round(flops / (g_ms * 1e-3) / 1e12, 1),
                     "frac_fp4": round(flops / (g_ms * 1e-3) / 1e12 / fp4_peak, 4),
                     "traffic": gemm_traffic(wl_name, M)},
            "quantize": {"ms": round(q_ms, 4), "GB/s": round(q_gbs, 1),
                         "frac_hbm": round(q_gbs / peaks["hbm_gbs"], 4)}}


def sustained_tflops(peaks):
    """The bf16 figure measured as a seconds-long loop under the power cap (the burst
    figure when the peaks file has none)."""
    return peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])


def linears_roofline_ms(synth, rows_x, rows_ctx, bits, peaks, sustained=False):
    """Tensor-core floor of one block's eight linears: each linear's FLOPs at the FP4
    (W4A4) or FP8 (W4A8) dense peak, the peaks being the measured bf16 burst (or, with
    `sustained`, the bf16 loop under the power cap) x the nominal dtype ratio."""
    bf16 = sustained_tflops(peaks) if sustained else peaks["bf16_tflops"]
    fp4 = bf16 * FP4_OVER_BF16 * 1e12
    fp8 = bf16 * FP8_OVER_BF16 * 1e12
    t = 0.0
    for i, (name, N, K, src) in enumerate(synth.BLOCK_LINEARS):
        rows = rows_x if src == "x" else rows_ctx
        t += 2.0 * rows * N * K / (fp8 if (bits >> i) & 1 else fp4)
    return t * 1e3


def bench_ffn(args, ops, synth, dev, stream, world, rank, peaks):
    """The block's FFN at 720p / 81 frames (M = 75600, dim 5120, hidden 13824) with the
    hidden activation kept MX-quantized (mxq_ffn: quantize, FFN-up GEMM whose epilogue
    applies GELU and quantizes, FFN-down GEMM), FFN-down in W4A4 or W4A8.  Beside it,
    for comparison only, the unfused pipeline: mxq_linear, torch's GELU on the bf16
    hidden activation, mxq_linear."""
    c = synth.BLOCK_720P
    M = c["M"]
    names = [n for n, *_ in synth.BLOCK_LINEARS]
    i_up, i_dn = names.index("ffn_up"), names.index("ffn_down")
    ws, bs = synth.block_weights(c["seed"], device=dev)
    up, down = ops.quantize_weight(ws[i_up], bias=bs[i_up]), ops.quantize_weight(ws[i_dn], bias=bs[i_dn])
    del ws, bs
    K, H, N2 = up.K, up.N, down.N
    x = synth.activation(M, K, "normal", seed=replica_seed(c["seed"] * 100 + i_up, rank), device=dev,
                         outlier_frac=0.01, outlier_scale=30.0)
    y = torch.empty((M, N2), dtype=torch.bfloat16, device=dev)
    flops = 2.0 * M * (K * H + H * N2)
    sus = sustained_tflops(peaks) / peaks["bf16_tflops"]  # sustained / burst
    fp4 = peaks["bf16_tflops"] * FP4_OVER_BF16 * 1e12
    fp8 = peaks["bf16_tflops"] * FP8_OVER_BF16 * 1e12
    iters = max(3, args.steps // 10)
    res = {"workload": "Wan-A14B FFN at 720p: M=%d, %d -> %d -> %d, FFN-up W4A4 (%.2f TFLOP)" % (
        M, K, H, N2, flops / 1e12)}
    for down_fmt in ("e2m1", "e4m3"):
        wsb = torch.empty(ops.ffn_workspace_bytes(M, K, H, "e2m1", down_fmt), dtype=torch.uint8, device=dev)
        fn = lambda f=down_fmt, w=wsb: ops.ffn(x, up, down, "e2m1", f, workspace=w, out=y)  # noqa: E731
        for _ in range(2):
            fn()
        with ClockSampler(dev.index) as clk:
            ms = time_loop(fn, iters, stream)
        ms = max_over_ranks(ms, world)
        roof = (2.0 * M * K * H / fp4 + 2.0 * M * H * N2 / (fp8 if down_fmt == "e4m3" else fp4)) * 1e3
        res["fused_down_" + down_fmt] = {"ms": round(ms, 3), "TFLOP/s": round(job_tflops(flops, ms, world), 1),
                                         "roofline_ms": round(roof, 3), "frac": round(roof / ms, 4),
                                         "frac_sustained": round(roof / sus / ms, 4),
                                         "launches": 3, "path": ops.last_path(), "clocks": clk.summary()}
        del wsb
    # unfused comparison (W4A4 down): bf16 hidden activation written, GELU by torch, read back
    hbuf = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    wsl = torch.empty(max(ops.workspace_bytes(M, H, K, "e2m1"), ops.workspace_bytes(M, N2, H, "e2m1")),
                      dtype=torch.uint8, device=dev)

    def unfused():
        ops.linear(x, up, "e2m1", workspace=wsl, out=hbuf)
        h = torch.nn.functional.gelu(hbuf)
        ops.linear(h, down, "e2m1", workspace=wsl, out=y)

    for _ in range(2):
        unfused()
    ms = max_over_ranks(time_loop(unfused, iters, stream), world)
    res["unfused_down_e2m1"] = {"ms": round(ms, 3), "TFLOP/s": round(job_tflops(flops, ms, world), 1),
                                "bf16_hidden_bytes_round_trip": 2 * M * H * 2 * 2,
                                "note": "comparison only: includes torch's GELU kernel"}
    if ops.poll_status() != 0:
        raise RuntimeError("device status set during the FFN measurement")
    return res


def bench_transform(args, ops, synth, dev, stream, world, rank, peaks, x, w, b):
    """The transform_on path on the headline workload: quantizer with per-channel smoothing
    and a block Hadamard rotation (32 or 128), and the linear built on it."""
    M, K = x.shape
    N = w.shape[0]
    from fp8_mixed_precision_mxq_b200 import policy
    s, inv_s = policy.smoothquant_scales(x, w, 0.5)  # SmoothQuant's scales, from the library
    flops = 2.0 * M * N * K
    qbytes = quant_bytes(M, K, "e2m1") + K * 4
    iters = max(3, args.steps // 4)
    codes = torch.empty(ops.codes_bytes(M, K, "e2m1"), dtype=torch.uint8, device=dev)
    sf = torch.empty(ops.sf_bytes(M, K), dtype=torch.uint8, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(ops.workspace_bytes(M, N, K, "e2m1"), dtype=torch.uint8, device=dev)
    res = {"workload": "%s (M=%d K=%d N=%d) W4A4, SmoothQuant scales (alpha 0.5) + block Hadamard" % (
        args.workload, M, K, N)}
    for block in (32, 128):
        qw = ops.quantize_weight_transformed(w, bias=b, block=block, mul=s)
        fq = lambda blk=block: ops.quantize_act_transformed(x, "e2m1", blk, inv_s, codes=codes, sf=sf)  # noqa: E731
        fl = lambda blk=block, q=qw: ops.linear_transformed(x, q, "e2m1", blk, inv_s, workspace=ws, out=y)  # noqa
        # the quantizer alone first (50 launches after a short probe), then the linear
        fq()
        q_ms, q_stats = time_kernel(fq, stream, idle_s=QUANT_IDLE_S)
        q_ms = max_over_ranks(q_ms, world)
        for _ in range(2):
            fl()
        l_ms = max_over_ranks(time_loop(fl, iters, stream), world)
        res["hadamard%d" % block] = {
            "quantize_ms": round(q_ms, 4), "quantize_GB/s": round(qbytes / (q_ms * 1e-3) / 1e9, 1),
            "quantize_frac_hbm": round(qbytes / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "quantize_launch_ms": q_stats,
            "linear_ms": round(l_ms, 4), "linear_TFLOP/s": round(job_tflops(flops, l_ms, world), 1)}
    if ops.poll_status() != 0:
        raise RuntimeError("device status set during the transform measurement")
    return res


def bench_lowrank(args, ops, synth, dev, stream, world, rank, peaks, x, b):
    """The SVDQuant low-rank branch on the headline workload: the linear with a rank-r bf16
    branch in the same accumulator, r = 64 and 128.  u = x . l1t^T and x's MX codes come
    from one kernel that reads x once (mxq_gemm_bf16_quant_a), timed alone against HBM."""
    c = synth.WORKLOADS[args.workload]
    M, K, N = x.shape[0], c["K"], c["N"]
    iters = max(3, args.steps // 4)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    res = {"workload": "%s (M=%d K=%d N=%d) W4A4 + bf16 rank-r branch" % (args.workload, M, K, N)}
    for r in (64, 128):
        l1t, l2t, resid = synth.lowrank_weight(N, K, r, seed=c["seed"], device=dev)
        qr = ops.quantize_weight(resid, bias=b)
        ws = torch.empty(ops.lowrank_workspace_bytes(M, N, K, "e2m1", r), dtype=torch.uint8, device=dev)
        fn = lambda q=qr, a=l1t, c2=l2t, w=ws: ops.linear_lowrank(x, q, a, c2, "e2m1", workspace=w, out=y)  # noqa
        for _ in range(2):
            fn()
        ms = max_over_ranks(time_loop(fn, iters, stream), world)
        flops = 2.0 * M * N * K + 2.0 * M * r * (K + N)
        res["rank%d" % r] = {"ms": round(ms, 4), "TFLOP/s": round(job_tflops(flops, ms, world), 1),
                             "branch_flop_share": round(2.0 * M * r * (K + N) / flops, 4), "path": ops.last_path()}
        # the fused u + quantizer kernel alone: x in, codes + scales + u out (HBM-bound)
        u = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
        xc = ws[: ops.codes_bytes(M, K, "e2m1")]
        off = (ops.codes_bytes(M, K, "e2m1") + 255) // 256 * 256
        xs = ws[off: off + ops.sf_bytes(M, K)]
        fq = lambda a=l1t, u=u, xc=xc, xs=xs: ops.gemm_bf16_quant_a(x, a, "e2m1", out=u, codes=xc, sf=xs)  # noqa
        fq()
        q_ms, q_stats = time_kernel(fq, stream, idle_s=QUANT_IDLE_S)
        q_ms = max_over_ranks(q_ms, world)
        qb = quant_bytes(M, K, "e2m1") + 2 * M * r + 2 * r * K
        res["rank%d" % r]["u_and_quantize"] = {
            "ms": round(q_ms, 4), "GB/s": round(qb / (q_ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(qb / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4), "bytes": qb,
            "launch_ms": q_stats, "path": ops.last_path()}
        del ws, u
    if ops.poll_status() != 0:
        raise RuntimeError("device status set during the low-rank measurement")
    return res


def bench_block(args, ops, synth, dev, stream, world, rank, peaks):
    """One DiT block's eight linears at 720p / 81 frames (M = 75600, text context 512)
    through the block entry point, under the three precision masks."""
    c = synth.BLOCK_720P
    M, ctx = c["M"], c["ctx"]
    ws, bs = synth.block_weights(c["seed"], device=dev)
    qws = [ops.quantize_weight(w, bias=b) for w, b in zip(ws, bs)]
    del ws, bs
    xs = synth.block_inputs(M, seed=replica_seed(c["seed"], rank), device=dev, ctx=ctx)
    rows = [x.shape[0] for x in xs]
    outs = [torch.empty((r, w.N), dtype=torch.bfloat16, device=dev) for r, w in zip(rows, qws)]
    wsb = torch.empty(ops.block_workspace_bytes(qws, rows, 0xFF), dtype=torch.uint8, device=dev)
    flops = synth.block_flops(M, ctx)
    iters = max(3, args.steps // 10)
    res = {"workload": "one Wan-A14B DiT block's 8 linears, M=%d video + %d text tokens (%.2f TFLOP)" % (
        M, ctx, flops / 1e12)}
    for name, bits in synth.BLOCK_MASKS.items():
        fn = lambda bits=bits: ops.dit_block_linears(qws, xs, bits, workspace=wsb, outs=outs)  # noqa: E731
        for _ in range(2):
            fn()
        with ClockSampler(dev.index) as clk:
            ms = time_loop(fn, iters, stream)
        ms = max_over_ranks(ms, world)
        roof = linears_roofline_ms(synth, M, ctx, bits, peaks)
        roof_s = linears_roofline_ms(synth, M, ctx, bits, peaks, sustained=True)
        res[name] = {"mask": "0x%02x" % bits, "ms": round(ms, 3),
                     "TFLOP/s": round(job_tflops(flops, ms, world), 1),
                     "roofline_ms": round(roof, 3), "frac": round(roof / ms, 4),
                     "frac_sustained": round(roof_s / ms, 4), "clocks": clk.summary()}
    # where the all-W4A4 block's time goes: each linear's quantizer and GEMM timed alone
    # (50 launches each) against that linear's FP4 floor
    fp4 = peaks["bf16_tflops"] * FP4_OVER_BF16 * 1e12
    per = []
    for i, (name, N, K, src) in enumerate(synth.BLOCK_LINEARS):
        rows_i = rows[i]
        xc = wsb[: ops.codes_bytes(rows_i, K, "e2m1")]
        off = (ops.codes_bytes(rows_i, K, "e2m1") + 255) // 256 * 256
        xsf = wsb[off: off + ops.sf_bytes(rows_i, K)]
        fq = lambda i=i, K=K, xc=xc, xsf=xsf: ops.quantize_act(xs[i], "e2m1", codes=xc, sf=xsf)  # noqa: E731
        fg = lambda i=i, K=K, r=rows_i, xc=xc, xsf=xsf: ops.gemm(xc, xsf, "e2m1", r, K, qws[i], out=outs[i])  # noqa
        fq()
        q_ms, _ = time_kernel(fq, stream)
        g_ms, _ = time_kernel(fg, stream)
        fl = 2.0 * rows_i * N * K
        per.append({"linear": name, "M": rows_i, "N": N, "K": K, "quantize_ms": round(max_over_ranks(q_ms, world), 4),
                    "gemm_ms": round(max_over_ranks(g_ms, world), 4),
                    "gemm_frac_fp4": round(fl / fp4 / (g_ms * 1e-3), 4)})
    res["all_w4a4_per_linear_alone"] = per
    if ops.poll_status() != 0:
        raise RuntimeError("device status set during the block measurement")
    return res


def profile_block(args, ops, synth, dev, stream):
    """Profiling mode for the block: one DiT block's eight linears at 720p under the
    all-W4A4 mask (overlapped quantizers), `steps` calls after the warm-up."""
    c = synth.BLOCK_720P
    ws, bs = synth.block_weights(c["seed"], device=dev)
    qws = [ops.quantize_weight(w, bias=b) for w, b in zip(ws, bs)]
    del ws, bs
    xs = synth.block_inputs(c["M"], seed=c["seed"], device=dev, ctx=c["ctx"])
    rows = [x.shape[0] for x in xs]
    outs = [torch.empty((r, w.N), dtype=torch.bfloat16, device=dev) for r, w in zip(rows, qws)]
    wsb = torch.empty(ops.block_workspace_bytes(qws, rows, 0x00), dtype=torch.uint8, device=dev)
    fn = lambda: ops.dit_block_linears(qws, xs, 0x00, workspace=wsb, outs=outs)  # noqa: E731
    for _ in range(args.warmup):
        fn()
    ms = time_loop(fn, args.steps, stream)
    status = ops.poll_status()
    print(json.dumps({"only": "block", "workload": "dit_block_720p all_w4a4", "M": c["M"], "ctx": c["ctx"],
                      "ms": round(ms, 4), "status": status, "path": ops.last_path()}))
    if status != 0:
        raise RuntimeError("device status %d" % status)


def bench_stack(args, ops, synth, dev, stream, world, rank, peaks):
    """The two-expert stack of 40 blocks at 480p / 81 frames: all 80 blocks' MXFP4
    weights resident, 8 random blocks per expert in W4A8; one timed unit is the forward
    of one expert through every linear of its 40 blocks."""
    c = synth.STACK_480P
    M, ctx, E, B = c["M"], c["ctx"], c["n_experts"], c["n_blocks"]
    mask = synth.expert_masks(E, B, c["n_w4a8"], seed=c["seed"])
    stack = []
    for e in range(E):
        blocks = []
        for blk in range(B):
            ws, bs = synth.block_weights(synth.stack_block_seed(e, blk), device=dev)
            blocks.append([ops.quantize_weight(w, bias=b) for w, b in zip(ws, bs)])
            del ws, bs
        stack.append(blocks)
    resident = sum(q.codes.numel() + q.sf.numel() for blocks in stack for blk in blocks for q in blk)
    xs = synth.block_inputs(M, seed=replica_seed(c["seed"], rank), device=dev, ctx=ctx)
    rows = [x.shape[0] for x in xs]
    outs = [torch.empty((r, w.N), dtype=torch.bfloat16, device=dev) for r, w in zip(rows, stack[0][0])]
    wsb = torch.empty(ops.block_workspace_bytes(stack[0][0], rows, 0xFF), dtype=torch.uint8, device=dev)
    bits = [[0xFF if mask[e, blk] else 0x00 for blk in range(B)] for e in range(E)]

    def forward(e):
        for blk in range(B):
            ops.dit_block_linears(stack[e][blk], xs, bits[e][blk], workspace=wsb, outs=outs)

    for e in range(E):
        forward(e)
    iters = max(2, args.steps // 50)
    flops = B * synth.block_flops(M, ctx)
    res = {"workload": "two experts x %d blocks, MXFP4 weights resident (%.1f GB), %d W4A8 blocks per expert, "
                       "M=%d video + %d text tokens; unit = one expert's forward (%.1f TFLOP)" % (
                           B, resident / 1e9, c["n_w4a8"], M, ctx, flops / 1e12)}
    for e in range(E):
        with ClockSampler(dev.index) as clk:
            ms = time_loop(lambda e=e: forward(e), iters, stream)
        ms = max_over_ranks(ms, world)
        roof = sum(linears_roofline_ms(synth, M, ctx, bits[e][blk], peaks) for blk in range(B))
        roof_s = sum(linears_roofline_ms(synth, M, ctx, bits[e][blk], peaks, sustained=True) for blk in range(B))
        res["expert%d" % e] = {"w4a8_blocks": [blk for blk in range(B) if bits[e][blk]], "ms": round(ms, 2),
                               "TFLOP/s": round(job_tflops(flops, ms, world), 1),
                               "roofline_ms": round(roof, 2), "frac": round(roof / ms, 4),
                               "frac_sustained": round(roof_s / ms, 4), "clocks": clk.summary()}
    if ops.poll_status() != 0:
        raise RuntimeError("device status set during the expert-stack measurement")
    return res


def bench_w4a8(args, ops, synth, dev, stream, world, rank, peaks):
    c = synth.WORKLOADS["ffn_down_720p_w4a8"]
    M, K, N = c["M"], c["K"], c["N"]
    x = synth.activation(M, K, c["act"], seed=replica_seed(c["seed"], rank), device=dev,
                         outlier_frac=c["outlier_frac"], outlier_scale=c["outlier_scale"])
    w = synth.weight(N, K, seed=c["seed"], device=dev)
    qw = ops.quantize_weight(w, bias=synth.bias(N, seed=c["seed"], device=dev))
    ws = torch.empty(ops.workspace_bytes(M, N, K, "e4m3", "qdq"), dtype=torch.uint8, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flops = 2.0 * M * N * K
    out = {"workload": "ffn_down_720p_w4a8: Wan2.2-A14B FFN-down, M=%d K=%d N=%d, E4M3 act (32-elem E8M0) x "
                       "MXFP4 weight" % (M, K, N)}
    iters = max(3, args.steps // 2)
    for mode in ("native", "qdq"):
        for _ in range(2):
            ops.linear(x, qw, "e4m3", mode=mode, workspace=ws, out=y)
        ms = max_over_ranks(time_loop(lambda: ops.linear(x, qw, "e4m3", mode=mode, workspace=ws, out=y), iters,
                                      stream), world)
        out[mode] = {"ms": round(ms, 4), "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1),
                     "path": ops.last_path()}
    xc = ws[: ops.codes_bytes(M, K, "e4m3")]
    off = (ops.codes_bytes(M, K, "e4m3") + 255) // 256 * 256
    xs = ws[off: off + ops.sf_bytes(M, K)]
    q_ms, q_stats = time_kernel(lambda: ops.quantize_act(x, "e4m3", codes=xc, sf=xs), stream, idle_s=QUANT_IDLE_S)
    q_ms = max_over_ranks(q_ms, world)
    g_ms = max_over_ranks(time_loop(lambda: ops.gemm(xc, xs, "e4m3", M, K, qw, out=y), iters, stream), world)
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    out["quantize_e4m3"] = {"ms": round(q_ms, 4), "GB/s": round(quant_bytes(M, K, "e4m3") / (q_ms * 1e-3) / 1e9, 1),
                            "frac_hbm": round(quant_bytes(M, K, "e4m3") / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                            "launch_ms": q_stats}
    out["gemm_mxf8f6f4"] = {"ms": round(g_ms, 4), "TFLOP/s": round(flops / (g_ms * 1e-3) / 1e12, 1),
                            "frac_fp8": round(flops / (g_ms * 1e-3) / 1e12 / fp8_peak, 4),
                            "peak_fp8": round(fp8_peak, 1)}
    # static per-tensor E4M3 activations (calibrated once, outside the timed region)
    scale = ops.absmax(x).item() / 448.0
    for _ in range(2):
        ops.linear_static(x, qw, scale, workspace=ws, out=y)
    s_ms = max_over_ranks(time_loop(lambda: ops.linear_static(x, qw, scale, workspace=ws, out=y), iters, stream),
                          world)
    sq_ms, sq_stats = time_kernel(lambda: ops.quantize_act_static(x, scale, codes=xc, sf=xs), stream,
                                  idle_s=QUANT_IDLE_S)
    sq_ms = max_over_ranks(sq_ms, world)
    out["static_e4m3"] = {"scale": scale, "linear_ms": round(s_ms, 4),
                          "linear_TFLOP/s": round(flops / (s_ms * 1e-3) / 1e12, 1),
                          "quantize_ms": round(sq_ms, 4),
                          "quantize_GB/s": round(quant_bytes(M, K, "e4m3") / (sq_ms * 1e-3) / 1e9, 1),
                          "quantize_frac_hbm": round(quant_bytes(M, K, "e4m3") / (sq_ms * 1e-3) / 1e9 /
                                                     peaks["hbm_gbs"], 4),
                          "quantize_launch_ms": sq_stats}
    if ops.poll_status() != 0:
        raise RuntimeError("device status set during the W4A8 measurement")
    return out


def run_reference(args):
    """The reference arm: the CPU oracle, on the host's CPU cores, on a bounded sample
    of the same workload per step.  Under torchrun only rank 0 runs it."""
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    c = synth.WORKLOADS[args.workload]
    M, K, N, fmt = c["M"], c["K"], c["N"], c["fmt"]
    cores = oracle.default_threads()
    # about 150 s of oracle work over the whole run, at least half a second per step
    per_step = max(0.5, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    if args.ref_step_seconds:
        per_step = args.ref_step_seconds
    for _ in range(args.warmup):
        cpu_gemm_rate(M, N, K, fmt, c["seed"], per_step / 2, cores)
    vals, rows = [], 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v_step, r_step, _ = cpu_gemm_rate(M, N, K, fmt, c["seed"], per_step, cores)
        vals.append(v_step)
        rows += r_step
    dt = time.perf_counter() - t0
    v = statistics.mean(vals)
    samples = {"cores": cores, "sample": "%d activation rows in all (about %.1f s per step) of the %dx%dx%d %s "
                                         "linear: quantize + fp64 GEMM on the dequantized operands, weight "
                                         "quantized beforehand, %d threads" % (rows, per_step, M, N, K, fmt, cores)}
    out = {"impl": "reference", "metric": "W4A4 MX linear TFLOP/s (fused dynamic MXFP4 activation quantize + "
                                          "tcgen05 mxf4 GEMM)",
           "value": v, "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(dt / max(1, args.steps) * 1e3, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "%s (CPU oracle on a bounded row sample per step)" % args.workload,
                      "M": M, "K": K, "N": N, "act_fmt": fmt},
           "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": samples["cores"], "kind": "oracle",
                            "sample": samples["sample"]},
           "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mxq", "reference"], default="mxq")
    ap.add_argument("--workload", default="ffn_up_720p_w4a4")
    ap.add_argument("--no-w4a8", dest="w4a8", action="store_false")
    ap.add_argument("--no-extra-linear", dest="extra_linear", action="store_false",
                    help="skip the 480p FFN-up (M=32760) measurement beside the headline")
    ap.add_argument("--no-transform", dest="transform", action="store_false",
                    help="skip the smoothing + Hadamard quantizer measurement")
    ap.add_argument("--no-lowrank", dest="lowrank", action="store_false",
                    help="skip the SVDQuant low-rank branch measurement")
    ap.add_argument("--no-ffn", dest="ffn", action="store_false",
                    help="skip the fused-FFN (M=75600) measurement")
    ap.add_argument("--no-block", dest="block", action="store_false",
                    help="skip the DiT-block (M=75600) measurement under the three masks")
    ap.add_argument("--no-stack", dest="stack", action="store_false",
                    help="skip the two-expert 40-block stack measurement")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=6.0,
                    help="seconds of CPU-oracle linear work per thread count")
    ap.add_argument("--ref-step-seconds", type=float, default=0.0,
                    help="reference arm: seconds of oracle work per step (default: about 150 s over the run)")
    ap.add_argument("--M", type=int, default=0, help="override the workload's row count (profiling)")
    ap.add_argument("--only", choices=["gemm", "quantize", "gelu_quant", "transform", "dequantize", "quantize_static",
                                       "gemm_bf16", "u_quantize", "block"], default=None,
                    help="profiling mode: launch only this kernel, --steps times")
    ap.add_argument("--rot-block", type=int, default=32, choices=[32, 128],
                    help="profiling mode: rotation block of the transform quantizer")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_mxq(args)


if __name__ == "__main__":
    main()
