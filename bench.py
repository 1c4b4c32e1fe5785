#!/usr/bin/env python
"""Benchmark of the B200 BitNet b1.58 BitLinear forward.

Headline workload (one "step"): the decode forward (RMSNorm + absmax int8
quant, ternary matmul, dequant) of the 70B-shaped layers K=8192->N=28672 and
K=28672->N=8192 at M = 1, 16 and 64 tokens each -- six forwards, bf16
activations with 0.1% x20 outlier channels, bf16 output, packed weights in
the tiled layout (converted once, offline), inputs resident in HBM, issued
as one bitnet_linear_forward_grouped call per step.  Every forward of a step
reads its own copy of the weights and the steps rotate over several such
sets (more than 1 GB of packed weights), so no step reads weights still in
L2.  The timed region (K steps) is repeated `--trials` times; the line
reports the median and the spread.

Besides the headline the line carries the roofline of the step's dominant
kernel, the end-to-end number through the C ABI with host buffers, a
per-configuration table for every workload of the suite (decode GB/s,
prefill int8 TOPS against the measured tensor-core rate), the measured int8
peak, the clocks seen during the timed regions, and the CPU oracle's rate.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle on
the same metric instead.  Under torchrun each rank runs an independent
replica (no data-path collective); timing is the max over ranks.
"""
import argparse
import ctypes
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BitLinear fwd: decode HBM GB/s & tok/s, prefill int8 TOPS (% of B200 peak)"
HEADLINE = "sweep_70b"
HEADLINE_MS = (1, 16, 64)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) of one launch of the headline's dominant kernel
# (the tiled decode matmul over the step's four M <= 16 forwards) from an
# ncu capture (summary under profiles/), valid only for the kernel source it
# was measured on (sha256 of csrc/gemv_tiled.cuh); reported as null otherwise.
GT_TRAFFIC = {"src_sha256": "bb301936c005a44543591601ed7d4b47cc9790fd15227512e5d5bff9186c5db6",
              "bytes_per_launch": 235698688 + 4319232}


# ------------------------------------------------------------------ helpers

def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def forward_bytes(M, N, K, x_bytes=2, y_bytes=2):
    """Algorithmic HBM bytes of one forward: x read, x_q written and read back,
    scales/row sums, packed weights, y written."""
    return M * K * x_bytes + 2 * M * K + 16 * M + 4 + N * K // 4 + M * N * y_bytes


def gemv_bytes(M, N, K, y_bytes=2):
    """Algorithmic bytes of the matmul kernel: packed weights, quantized
    activations, scales and row sums, s_w, y."""
    return N * K // 4 + M * K + 8 * M + 4 + M * N * y_bytes


def file_sha256(path):
    import hashlib
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def max_over_ranks(value, world, device=None):
    """Max of a float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step_per_rank, steps, world, max_ms):
    """Whole-job GB/s: the bytes all ranks processed over the slowest rank's time."""
    return bytes_per_step_per_rank * steps * world / (max_ms * 1e-3) / 1e9


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, period_s=0.001, window=""):
        self.index, self.period, self.window = index, period_s, window
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok and self._t is None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()
            self._t = None

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml unavailable"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "source": "nvml", "window": self.window}


def case_problems(name, ms=None):
    from ternary_quantized_linear_b200 import workloads
    case = workloads.CASE_BY_NAME[name]
    probs = [p for p in workloads.all_problems(case) if ms is None or p[3] in ms]
    return case, probs


# --------------------------------------------------------------- CPU oracle

def time_oracle(case_name, probs, budget_s, max_steps=None, threads=1):
    """Run the CPU oracle on the problems (cycling, one forward at a time)
    until budget_s is spent or max_steps forwards ran, its integer matmul on
    `threads` threads.  Returns (bytes, seconds, forwards, threads in effect)."""
    import oracle
    from ternary_quantized_linear_b200 import workloads
    threads = oracle.set_threads(threads)
    case = workloads.CASE_BY_NAME[case_name]
    wcache, prepared = {}, []
    for si, K, N, M in probs:
        if si not in wcache:
            W = workloads.weights(case, si)
            s_w, _ = oracle.weight_scale(W)
            W_p, _ = oracle.quantize_pack(W, s_w)
            wcache[si] = (W_p, s_w)
            del W
        prepared.append((workloads.activations(case, si, M), wcache[si], K, N, M))
    total_b, total_s, units = 0, 0.0, 0
    t_start = time.perf_counter()
    i = 0
    while True:
        x, (W_p, s_w), K, N, M = prepared[i % len(prepared)]
        t0 = time.perf_counter()
        oracle.linear_forward(x, None, workloads.DEFAULT_EPS, W_p, s_w, K)
        total_s += time.perf_counter() - t0
        total_b += forward_bytes(M, N, K)
        units += 1
        i += 1
        if max_steps is not None and units >= max_steps:
            break
        if max_steps is None and time.perf_counter() - t_start >= budget_s:
            break
    return total_b, total_s, units, threads


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return 0
    case, probs = case_problems(HEADLINE, (1,))
    # one step here is one M = 1 forward of the headline's layers (the
    # oracle's full step would take minutes); warm-up untimed
    time_oracle(HEADLINE, probs, 0, max_steps=max(args.warmup, 1))
    b, s, units, threads = time_oracle(HEADLINE, probs, 0, max_steps=args.steps)
    gbs = b / s / 1e9
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * s / units, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": HEADLINE + ": " + case.description, "x_dtype": "bf16",
                   "y_dtype": "bf16"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{units} single forwards (M = 1) of the 70B-shaped layers, "
                                   "cycling, plain C oracle, 1 thread"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------- GPU path

class DecodeWorkload:
    """Decode forwards of one case on tiled weights: `rot` rotation sets,
    each forward of each set with its own weight copy, one grouped call per
    set (= one step)."""

    def __init__(self, tql, workloads, case_name, ms, rot, device, tiled_cache):
        import numpy as np
        import torch
        self.case, self.probs = case_problems(case_name, ms)
        self.rot = rot
        self.sets = []
        base = {}
        for si, (K, N) in enumerate(self.case.shapes):
            if not any(p[0] == si for p in self.probs):
                continue
            key = (case_name, si)
            if key not in tiled_cache:
                W = torch.from_numpy(workloads.weights(self.case, si)).to(device)
                W_p, s_w = tql.bitnet_quantize_pack_weights(W)
                del W
                tiled_cache[key] = (tql.bitnet_tile_weights(W_p), s_w)
                del W_p
            base[si] = tiled_cache[key]
        for r in range(rot):
            items = []
            for si, K, N, M in self.probs:
                Wt, s_w = base[si]
                Wc = tql.TiledWeights(Wt.data.clone(), Wt.N, Wt.K)
                xh = workloads.activations(self.case, si, M)
                x = torch.from_numpy(xh.view(np.int16).copy()).view(torch.bfloat16).to(device)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
                items.append((x, None, workloads.DEFAULT_EPS, Wc, s_w, y))
            arr, count = tql.grouped_problems(items)
            nb = tql.bitnet_linear_forward_grouped_workspace_bytes(arr, count)
            ws = torch.empty(nb, dtype=torch.uint8, device=device)
            self.sets.append({"items": items, "arr": arr, "count": count, "ws": ws})
        self.weight_bytes = sum(it[3].data.numel() for s in self.sets for it in s["items"])

    def step_bytes(self):
        return sum(forward_bytes(M, N, K) for _, K, N, M in self.probs)

    def tokens(self):
        return sum(M for _, _, _, M in self.probs)


def grouped_call(lib, tql, st, phases, stream_handle):
    rc = lib.bitnet_linear_forward_grouped(st["count"], ctypes.cast(st["arr"], ctypes.c_void_p),
                                           ctypes.c_void_p(st["ws"].data_ptr()),
                                           st["ws"].numel(), phases, stream_handle)
    if rc != 0:
        raise RuntimeError(f"bitnet_linear_forward_grouped: {tql.bitnet_status_string(rc)}")


def timed_graph_steps(torch, stream, calls, steps, warmup, trials):
    """calls: R callables (one step each, taking a stream handle).  Captures
    the R steps back to back in one CUDA graph (and single-step graphs for a
    remainder), runs `warmup` untimed steps, then times exactly `steps` steps
    `trials` times with CUDA events on `stream`.  Returns ms per trial."""
    R = len(calls)
    P = ctypes.c_void_p
    with torch.cuda.stream(stream):
        for c in calls:
            c(P(stream.cuda_stream))
        stream.synchronize()
        rotation = torch.cuda.CUDAGraph()
        with torch.cuda.graph(rotation, stream=stream):
            for c in calls:
                c(P(torch.cuda.current_stream().cuda_stream))
        singles = []
        for c in calls[:steps % R]:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                c(P(torch.cuda.current_stream().cuda_stream))
            singles.append(g)

        def run(k):
            for _ in range(k // R):
                rotation.replay()
            for g in singles[:k % R]:
                g.replay()

        run(max(warmup, 1))
        stream.synchronize()
        out = []
        for _ in range(trials):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run(steps)
            e1.record(stream)
            stream.synchronize()
            out.append(e0.elapsed_time(e1))
    del rotation, singles
    return out


def run_ours(args):
    import numpy as np
    import torch

    rank, world, local_rank = env_rank()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    import ternary_quantized_linear_b200 as tql
    from ternary_quantized_linear_b200 import build as tql_build
    from ternary_quantized_linear_b200 import workloads

    tql_build.build()
    lib = tql.load_library()
    stream = torch.cuda.Stream(device=device)
    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tiled_cache = {}

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local_rank])

    # ---- headline: the 70B decode step, R rotation sets of six forwards
    head = DecodeWorkload(tql, workloads, HEADLINE, HEADLINE_MS, args.rotations, device,
                          tiled_cache)
    torch.cuda.synchronize()
    calls = [lambda h, st=st: grouped_call(lib, tql, st, tql.BITNET_PHASE_ALL, h)
             for st in head.sets]
    clocks = ClockSampler(local_rank, window="the headline's warm-up and timed trials, the "
                                             "kernel timing and the per-config timings")
    clocks.start()
    barrier()
    trial_ms = timed_graph_steps(torch, stream, calls, args.steps, args.warmup, args.trials)
    barrier()
    med_ms = statistics.median(trial_ms)
    max_ms = max_over_ranks(med_ms, world, device)
    sb = head.step_bytes()
    value = job_throughput(sb, args.steps, world, max_ms)
    trial_gbs = sorted(sb * args.steps / (t * 1e-3) / 1e9 for t in trial_ms)
    ms_per_step = max_ms / args.steps
    # kernel launches per step: one activation-quant launch for all six
    # forwards, the tiled decode matmul for the four M <= 16 forwards and its
    # fixup of split row blocks (these shapes split some), and a tcgen05
    # launch for each M = 64 forward (the launch list under profiles/ shows
    # the same count)
    n_big = sum(1 for p in head.probs if p[3] > 16)
    launches_per_step = 3 + n_big

    # ---- roofline: the tiled decode matmul of the four M <= 16 forwards
    # (the dominant kernel: 4 x 58.7 MB of the step's 6 x 58.7 MB), timed
    # alone as the matmul phase of a group holding just those forwards.
    small_sets = []
    for st in head.sets:
        items = [it for it in st["items"] if it[0].shape[0] <= 16]
        arr, count = tql.grouped_problems(items)
        small_sets.append({"items": items, "arr": arr, "count": count, "ws": st["ws"]})
    with torch.cuda.stream(stream):   # quantize once into each set's workspace
        for st in small_sets:
            grouped_call(lib, tql, st, tql.BITNET_PHASE_QUANTIZE, ctypes.c_void_p(stream.cuda_stream))
        stream.synchronize()
    mm_calls = [lambda h, st=st: grouped_call(lib, tql, st, tql.BITNET_PHASE_MATMUL, h)
                for st in small_sets]
    k_ms = timed_graph_steps(torch, stream, mm_calls, args.steps, args.warmup, args.trials)
    gt_ms = statistics.median(k_ms) / args.steps
    gt_b = sum(gemv_bytes(M, N, K) for _, K, N, M in head.probs if M <= 16)
    achieved = gt_b / (gt_ms * 1e-3) / 1e9
    sha = file_sha256(os.path.join(ROOT, "ternary_quantized_linear_b200", "csrc",
                                   "gemv_tiled.cuh"))
    traffic = GT_TRAFFIC["bytes_per_launch"] if GT_TRAFFIC["src_sha256"] == sha else None
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                "kernel": "ternary_gemv_tiled_kernel, one launch over the step's four M <= 16 "
                          "forwards (matmul + fused dequant)",
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
                "algorithmic_bytes_per_launch": gt_b,
                "avg_launch_us": round(1e3 * gt_ms, 2),
                "how": "CUDA events around back-to-back CUDA-graph replays of the matmul "
                       f"phase alone over {args.rotations} rotating weight sets, median of "
                       f"{args.trials} trials of {args.steps} launches"}

    # ---- int8 tensor-core rate (the prefill roofline's denominator)
    i8 = measure_int8_peak(tql, torch, stream)

    # ---- per-configuration table
    per_config = []
    if not args.no_configs:
        per_config = measure_configs(args, tql, lib, workloads, torch, stream, device, hbm_peak,
                                     i8, tiled_cache, head, value, gt_ms, gt_b)
    clocks.stop()

    # ---- end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, tql, lib, torch, stream, device, head, world, barrier)

    weight_pack = None
    if not args.no_weight_pack:
        try:
            weight_pack = measure_weight_pack(args, tql, workloads, torch, stream, device,
                                              hbm_peak)
        except Exception as exc:  # noqa: BLE001 -- report, keep the line
            weight_pack = {"error": str(exc)}

    # ---- CPU baseline (rank 0, one GPU only): the oracle on a bounded
    # sample of the headline workload
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        _, probs1 = case_problems(HEADLINE, (1,))
        b, s, units, threads = time_oracle(HEADLINE, probs1, args.cpu_budget)
        cpu = {"value": b / s / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{units} single forwards (M = 1) of the two 70B-shaped layers, "
                         f"cycling, plain C oracle, {threads} thread(s), {s:.1f} s"}
        ncores = os.cpu_count() or 1
        b, s, units, threads = time_oracle(HEADLINE, probs1, args.cpu_budget / 2, threads=ncores)
        cpu["all_cores"] = {"value": b / s / 1e9, "unit": "GB/s", "cores": threads,
                            "sample": f"{units} forwards, integer matmul on {threads} "
                                      f"thread(s), {s:.1f} s"}

    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic",
            "config": {"workload": HEADLINE + ": " + head.case.description,
                       "problems": [[K, N, M] for _, K, N, M in head.probs],
                       "x_dtype": "bf16", "y_dtype": "bf16", "weights": "tiled layout",
                       "l2": f"inputs larger than L2: {args.rotations} rotating sets, every "
                             f"forward with its own weight copy, "
                             f"{head.weight_bytes / 1e6:.0f} MB of packed weights",
                       "launch": "one bitnet_linear_forward_grouped call per step; the R "
                                 "rotation steps captured back to back in one CUDA graph",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "trials": {"count": args.trials, "median_gbs": round(statistics.median(trial_gbs), 1),
                       "min_gbs": round(trial_gbs[0], 1), "max_gbs": round(trial_gbs[-1], 1)},
            "tok_s": round(world * head.tokens() * args.steps / (max_ms * 1e-3), 1),
            "roofline": roofline,
            "int8_peak": i8,
            "per_config": per_config,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(),
            "weight_pack": weight_pack,
        }
        print(json.dumps(line), flush=True)
    return 0


def measure_int8_peak(tql, torch, stream):
    """Dense int8 tensor-core rate: one CTA per SM issuing 128x256x32
    tcgen05 MMAs back to back (A in shared memory, and in tensor memory as
    the forward's kernels use it), timed with CUDA events."""
    sms = torch.cuda.get_device_properties(stream.device).multi_processor_count
    res = {}
    for name, tmem in (("a_smem", False), ("a_tmem", True)):
        iters = 20000
        with torch.cuda.stream(stream):
            tql.bitnet_selftest_mma_i8(1000, sms, tmem, stream=stream)
            stream.synchronize()
            best = None
            for _ in range(3):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                ops = tql.bitnet_selftest_mma_i8(iters, sms, tmem, stream=stream)
                e1.record(stream)
                stream.synchronize()
                ms = e0.elapsed_time(e1)
                best = ms if best is None else min(best, ms)
        res[name] = round(ops / (best * 1e-3) / 1e12, 1)
    code, _ = tql.bitnet_device_status(reset=False, stream=stream)
    return {"tops": max(res.values()), "a_smem_tops": res["a_smem"],
            "a_tmem_tops": res["a_tmem"], "source": "measured",
            "how": f"bitnet_selftest_mma_i8: {sms} CTAs x 20000 tcgen05.mma kind::i8 "
                   "128x256x32, best of 3, CUDA events", "status_ok": code == tql.BITNET_OK,
            "spec_tops": 4500.0}


def measure_configs(args, tql, lib, workloads, torch, stream, device, hbm_peak, i8, tiled_cache,
                    head, head_value, head_gt_ms, head_gt_b):
    """One entry per workload of the suite: decode GB/s (and the roofline of
    its decode matmul launch), prefill int8 TOPS against the measured rate."""
    import numpy as np
    out = []
    P = ctypes.c_void_p
    steps, trials = max(6, args.steps // 2), max(3, args.trials // 2)

    # tiny: one fp32 forward through the plain C-ABI call
    x, W = workloads.tiny_inputs()
    W_p, s_w = tql.bitnet_quantize_pack_weights(torch.from_numpy(W).to(device))
    xd = torch.from_numpy(x).to(device)
    y = torch.empty((16, 512), dtype=torch.float32, device=device)
    ws = torch.empty(tql.bitnet_linear_forward_workspace_bytes(16, 512, 256), dtype=torch.uint8,
                     device=device)

    def tiny_call(h):
        rc = lib.bitnet_linear_forward(P(xd.data_ptr()), tql.BITNET_F32, None,
                                       ctypes.c_float(1e-5), P(W_p.data_ptr()),
                                       P(s_w.data_ptr()), 16, 512, 256, P(y.data_ptr()),
                                       tql.BITNET_F32, P(ws.data_ptr()), ws.numel(), h)
        if rc != 0:
            raise RuntimeError(tql.bitnet_status_string(rc))

    t = statistics.median(timed_graph_steps(torch, stream, [tiny_call], 50, 5, trials)) / 50
    b = forward_bytes(16, 512, 256, 4, 4)
    out.append({"config": "tiny", "problems": [[256, 512, 16]], "us_per_forward": round(1e3 * t, 2),
                "gbs": round(b / (t * 1e-3) / 1e9, 1), "note": "fp32 in/out, L2-resident, "
                "launch-bound (two launches of a 65 KB problem)"})

    # decode configs: grouped steps on tiled weights
    for name in ("decode_bitnet3b", "decode_llama3_8b"):
        wl = DecodeWorkload(tql, workloads, name, None, 6, device, tiled_cache)
        calls = [lambda h, st=st: grouped_call(lib, tql, st, tql.BITNET_PHASE_ALL, h)
                 for st in wl.sets]
        ms = statistics.median(timed_graph_steps(torch, stream, calls, steps, 3, trials)) / steps
        mm_calls = [lambda h, st=st: grouped_call(lib, tql, st, tql.BITNET_PHASE_MATMUL, h)
                    for st in wl.sets]
        mm = statistics.median(timed_graph_steps(torch, stream, mm_calls, steps, 3, trials)) / steps
        gb = sum(gemv_bytes(M, N, K) for _, K, N, M in wl.probs)
        out.append({"config": name, "problems": [[K, N, M] for _, K, N, M in wl.probs],
                    "step_us": round(1e3 * ms, 2),
                    "gbs": round(wl.step_bytes() / (ms * 1e-3) / 1e9, 1),
                    "tok_s": round(wl.tokens() / (ms * 1e-3), 1),
                    "matmul_us": round(1e3 * mm, 2),
                    "matmul_frac_of_hbm": round(gb / (mm * 1e-3) / 1e9 / hbm_peak, 4)})
        del wl
        torch.cuda.empty_cache()

    # prefill: the tcgen05 kernel on tiled weights
    def prefill(name, ms_list):
        case = workloads.CASE_BY_NAME[name]
        rows = []
        for si, (K, N) in enumerate(case.shapes):
            key = (name, si)
            if key not in tiled_cache:
                Wd = torch.from_numpy(workloads.weights(case, si)).to(device)
                Wp, sw = tql.bitnet_quantize_pack_weights(Wd)
                del Wd
                tiled_cache[key] = (tql.bitnet_tile_weights(Wp), sw)
            Wt, sw = tiled_cache[key]
            for M in ms_list:
                xh = workloads.activations(case, si, M)
                xs = torch.from_numpy(xh.view(np.int16).copy()).view(torch.bfloat16).to(device)
                yy = torch.empty((M, N), dtype=torch.bfloat16, device=device)
                items = [(xs, None, 1e-5, Wt, sw, yy)]
                arr, count = tql.grouped_problems(items)
                nb = tql.bitnet_linear_forward_grouped_workspace_bytes(arr, count)
                wsp = torch.empty(nb, dtype=torch.uint8, device=device)
                st = {"items": items, "arr": arr, "count": count, "ws": wsp}
                n_it = 4 if M >= 4096 else 10
                f = statistics.median(timed_graph_steps(
                    torch, stream, [lambda h: grouped_call(lib, tql, st, tql.BITNET_PHASE_ALL, h)],
                    n_it, 2, trials)) / n_it
                mm = statistics.median(timed_graph_steps(
                    torch, stream,
                    [lambda h: grouped_call(lib, tql, st, tql.BITNET_PHASE_MATMUL, h)],
                    n_it, 2, trials)) / n_it
                ops = 2.0 * M * N * K
                tops = ops / (mm * 1e-3) / 1e12
                rows.append({"K": K, "N": N, "M": M, "forward_us": round(1e3 * f, 2),
                             "gemm_us": round(1e3 * mm, 2), "gemm_tops": round(tops, 1),
                             "forward_tops": round(ops / (f * 1e-3) / 1e12, 1),
                             "frac_of_measured_int8": round(tops / i8["tops"], 4),
                             "frac_of_4500_spec": round(tops / 4500.0, 4)})
                del xs, yy, wsp, st
        return rows

    pre = prefill("prefill_llama3_8b", (512, 2048, 8192))
    out.append({"config": "prefill_llama3_8b", "shapes": pre,
                "tops_mean": round(statistics.mean(r["gemm_tops"] for r in pre), 1),
                "frac_of_measured_int8_mean": round(statistics.mean(
                    r["frac_of_measured_int8"] for r in pre), 4)})
    pre70 = prefill(HEADLINE, (1024, 4096))
    out.append({"config": HEADLINE, "decode": {
        "problems": [[K, N, M] for _, K, N, M in head.probs], "gbs": round(head_value, 1),
        "tiled_gemv_us": round(1e3 * head_gt_ms, 2),
        "tiled_gemv_frac_of_hbm": round(head_gt_b / (head_gt_ms * 1e-3) / 1e9 / hbm_peak, 4)},
        "prefill": pre70,
        "prefill_tops_mean": round(statistics.mean(r["gemm_tops"] for r in pre70), 1)})
    return out


def measure_e2e(args, tql, lib, torch, stream, device, head, world, barrier):
    """The headline step through the public C-ABI call with host buffers:
    every step uploads its six inputs from pinned host memory, makes the
    grouped call and downloads its six outputs; uploads, calls and downloads
    run on three streams ordered per rotation set by events, so step i's
    upload overlaps step i-1's call and download.  Device-timed."""
    P = ctypes.c_void_p
    R = len(head.sets)
    e2e_sets = []
    for st in head.sets:
        xs = [tuple(it[0].shape) for it in st["items"]]
        ys = [tuple(it[5].shape) for it in st["items"]]

        def packed(shapes):
            offs, n = [], 0
            for s in shapes:
                offs.append(n)
                n += -(-s[0] * s[1] // 64) * 64
            return offs, n

        xo, xn = packed(xs)
        yo, yn = packed(ys)
        dx = torch.empty(xn, dtype=torch.bfloat16, device=device)
        dy = torch.empty(yn, dtype=torch.bfloat16, device=device)
        hx = torch.empty(xn, dtype=torch.bfloat16).pin_memory()
        hy = torch.empty(yn, dtype=torch.bfloat16).pin_memory()
        items = []
        for j, it in enumerate(st["items"]):
            n = xs[j][0] * xs[j][1]
            hx[xo[j]:xo[j] + n].view(xs[j]).copy_(it[0].cpu())
            xv = dx[xo[j]:xo[j] + n].view(xs[j])
            yv = dy[yo[j]:yo[j] + ys[j][0] * ys[j][1]].view(ys[j])
            items.append((xv, None, it[2], it[3], it[4], yv))
        arr, count = tql.grouped_problems(items)
        e2e_sets.append({"dx": dx, "dy": dy, "hx": hx, "hy": hy, "arr": arr, "count": count,
                         "ws": st["ws"], "items": items, "yo": yo})
    h2d = sum(it[0].numel() * 2 for it in head.sets[0]["items"])
    d2h = sum(it[5].numel() * 2 for it in head.sets[0]["items"])

    cu = ctypes.CDLL("libcuda.so.1")
    VP, U64, SZ = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_size_t
    h2d_copy, d2h_copy = cu.cuMemcpyHtoDAsync_v2, cu.cuMemcpyDtoHAsync_v2
    h2d_copy.argtypes = [U64, VP, SZ, VP]
    d2h_copy.argtypes = [VP, U64, SZ, VP]
    ev_create, ev_record, ev_destroy = cu.cuEventCreate, cu.cuEventRecord, cu.cuEventDestroy_v2
    ev_create.argtypes = [ctypes.POINTER(VP), ctypes.c_uint]
    ev_record.argtypes = [VP, VP]
    ev_destroy.argtypes = [VP]
    wait_ev = cu.cuStreamWaitEvent
    wait_ev.argtypes = [VP, VP, ctypes.c_uint]

    def ok(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what} returned CUDA driver error {rc}")

    s_up, s_dn = torch.cuda.Stream(device), torch.cuda.Stream(device)
    h_up, h_c, h_dn = VP(s_up.cuda_stream), VP(stream.cuda_stream), VP(s_dn.cuda_stream)
    events = []

    def new_event():
        e = VP()
        ok(ev_create(ctypes.byref(e), 2), "cuEventCreate")  # CU_EVENT_DISABLE_TIMING
        events.append(e)
        return e

    up = [new_event() for _ in range(R)]
    called = [new_event() for _ in range(R)]
    down = [new_event() for _ in range(R)]
    used = [False] * R
    plan = []
    for s in e2e_sets:
        plan.append((U64(s["dx"].data_ptr()), VP(s["hx"].data_ptr()),
                     SZ(s["dx"].numel() * 2), VP(s["hy"].data_ptr()), U64(s["dy"].data_ptr()),
                     SZ(s["dy"].numel() * 2), s["count"], ctypes.cast(s["arr"], P),
                     P(s["ws"].data_ptr()), s["ws"].numel()))
    call = lib.bitnet_linear_forward_grouped

    def step(r):
        dxp, hxp, nx, hyp, dyp, ny, count, arr_p, ws_p, nb = plan[r]
        if used[r]:
            ok(wait_ev(h_up, called[r], 0), "cuStreamWaitEvent")
        ok(h2d_copy(dxp, hxp, nx, h_up), "cuMemcpyHtoDAsync")
        ok(ev_record(up[r], h_up), "cuEventRecord")
        ok(wait_ev(h_c, up[r], 0), "cuStreamWaitEvent")
        if used[r]:
            ok(wait_ev(h_c, down[r], 0), "cuStreamWaitEvent")
        rc = call(count, arr_p, ws_p, nb, tql.BITNET_PHASE_ALL, h_c)
        if rc != 0:
            raise RuntimeError(tql.bitnet_status_string(rc))
        ok(ev_record(called[r], h_c), "cuEventRecord")
        ok(wait_ev(h_dn, called[r], 0), "cuStreamWaitEvent")
        ok(d2h_copy(hyp, dyp, ny, h_dn), "cuMemcpyDtoHAsync")
        ok(ev_record(down[r], h_dn), "cuEventRecord")
        used[r] = True

    def join():
        stream.wait_stream(s_up)
        stream.wait_stream(s_dn)

    times = []
    try:
        for i in range(args.warmup):
            step(i % R)
        join()
        torch.cuda.synchronize()
        barrier()
        for _ in range(max(3, args.trials // 2)):
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            s_up.wait_stream(stream)
            s_dn.wait_stream(stream)
            for i in range(args.steps):
                step(i % R)
            join()
            a1.record(stream)
            torch.cuda.synchronize()
            times.append(a0.elapsed_time(a1))
    finally:
        torch.cuda.synchronize()
        for e in events:
            ev_destroy(e)
    # the downloads hold what the device path computes for each set
    for r, s in enumerate(e2e_sets):
        if not used[r]:
            continue
        got = torch.cat([s["hy"][o:o + it[5].numel()] for o, it in zip(s["yo"], s["items"])])
        want = torch.cat([it[5].reshape(-1).cpu() for it in head.sets[r]["items"]])
        if not torch.equal(got.view(torch.int16), want.view(torch.int16)):
            raise RuntimeError(f"end-to-end outputs of set {r} differ from the device path")
    med = statistics.median(times)
    e2e_ms = max_over_ranks(med, world, device)
    return {"value": round(job_throughput(head.step_bytes(), args.steps, world, e2e_ms), 2),
            "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_ms / args.steps,
            "how": "per step: one pinned-host -> device copy of the six inputs, one "
                   "bitnet_linear_forward_grouped call (C ABI, eager), one device -> "
                   "pinned-host copy of the six outputs; uploads, calls and downloads on "
                   "three streams ordered per rotation set by events (copies and events "
                   "through the CUDA driver API); outputs checked against the device path; "
                   f"device-timed, median of {len(times)} trials"}


def measure_weight_pack(args, tql, workloads, torch, stream, device, hbm_peak):
    """bitnet_quantize_pack_weights on the BitNet-3B-shaped fp32 matrices
    (261 MB together, more than L2), cycled, outputs preallocated: the
    absmean pass reads W, the quantize pass reads it again and writes the
    packed codes (the scale must be known before any code is decided)."""
    case = workloads.CASE_BY_NAME["decode_bitnet3b"]
    mats = []
    for si, (K, N) in enumerate(case.shapes):
        W = torch.from_numpy(workloads.weights(case, si)).to(device)
        W_p = torch.empty((N, K // 4), dtype=torch.uint8, device=device)
        s_w = torch.empty((1,), dtype=torch.float32, device=device)
        nb = max(tql.bitnet_quantize_pack_weights_workspace_bytes(N, K), 256)
        ws = torch.empty(nb, dtype=torch.uint8, device=device)
        mats.append((W, W_p, s_w, ws, N, K))
    n = len(mats)
    reps = 10
    with torch.cuda.stream(stream):
        for i in range(3 * n):
            W, W_p, s_w, ws, _, _ = mats[i % n]
            tql.bitnet_quantize_pack_weights(W, W_p, s_w, ws, stream=stream)
        stream.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps * n)]
        for i in range(reps * n):
            W, W_p, s_w, ws, _, _ = mats[i % n]
            ev[i][0].record(stream)
            tql.bitnet_quantize_pack_weights(W, W_p, s_w, ws, stream=stream)
            ev[i][1].record(stream)
        stream.synchronize()
    per = []
    tot_b, tot_ms = 0, 0.0
    for j, (W, W_p, _, _, N, K) in enumerate(mats):
        ms = statistics.median(ev[i][0].elapsed_time(ev[i][1]) for i in range(j, reps * n, n))
        b = 2 * 4 * N * K + N * K // 4
        tot_b += b
        tot_ms += ms
        per.append({"N": N, "K": K, "us": round(1e3 * ms, 2),
                    "gbs": round(b / (ms * 1e-3) / 1e9, 1)})
    gbs = tot_b / (tot_ms * 1e-3) / 1e9
    return {"workload": "decode_bitnet3b weights, fp32, cycled", "matrices": per,
            "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / hbm_peak, 4),
            "bytes": "two reads of W (absmean, then quantize) + the packed write"}


def profile_kernel(args):
    """A small driver for an ncu capture of the roofline kernel: one rotation
    set of the headline's M <= 16 forwards (four forwards, each with its own
    copy of the tiled weights, 235 MB -- more than L2), two full grouped
    calls, then `--steps` calls of the matmul phase alone.  Prints one status
    line; no timing (numbers under a profiler are not bench values)."""
    import torch
    import ternary_quantized_linear_b200 as tql
    from ternary_quantized_linear_b200 import build as tql_build
    from ternary_quantized_linear_b200 import workloads
    tql_build.build()
    lib = tql.load_library()
    device = torch.device("cuda", 0)
    small = tuple(m for m in HEADLINE_MS if m <= 16)
    wl = DecodeWorkload(tql, workloads, HEADLINE, small, 1, device, {})
    st = wl.sets[0]
    h = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        grouped_call(lib, tql, st, tql.BITNET_PHASE_ALL, h)
    for _ in range(args.steps):
        grouped_call(lib, tql, st, tql.BITNET_PHASE_MATMUL, h)
    torch.cuda.synchronize()
    code, detail = tql.bitnet_device_status(reset=False)
    print(json.dumps({"profile_kernel": "done", "problems": [[K, N, M] for _, K, N, M in wl.probs],
                      "weight_bytes": wl.weight_bytes, "device_status": [int(code), int(detail)]}))
    return 0 if code == 0 else 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--trials", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--rotations", type=int, default=3)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--no-weight-pack", action="store_true")
    ap.add_argument("--profile-kernel", action="store_true",
                    help="only run the roofline kernel's launches (a driver for ncu)")
    args = ap.parse_args(argv)
    if args.profile_kernel:
        return profile_kernel(args)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
