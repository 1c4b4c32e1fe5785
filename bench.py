#!/usr/bin/env python
"""Benchmark of the B200 BitNet b1.58 BitLinear forward.

Workload (one "step"): the decode forward (RMSNorm + absmax int8 quant,
ternary matmul, dequant) of the BitNet-3B-shaped problems
K=3200->N=3200, 3200->8640 and 8640->3200 at M = 1, 4 and 16 tokens each
(nine problems), bf16 activations with 0.1% x20 outlier channels, bf16
output, inputs resident in HBM.  Weights rotate over several distinct copies
so that a step never reads weights that are still in L2.

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
WORKLOAD = "decode_bitnet3b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) of one grouped GEMV launch of this workload from
# an ncu capture (summary under profiles/), valid only for the kernel source
# it was measured on (sha256 of csrc/gemv.cuh); reported as null otherwise.
GEMV_TRAFFIC = {"src_sha256": "d5f0e05da58c50699640b00f12d8cc0c624cb952e6282a088a857f01a4bb1d51",
                "bytes_per_launch": 49537280}


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


def quant_bytes(M, K, x_bytes=2):
    return M * K * x_bytes + M * K + 8 * M


def problems():
    from ternary_quantized_linear_b200 import workloads
    case = workloads.CASE_BY_NAME[WORKLOAD]
    return case, list(workloads.all_problems(case))


def step_bytes(probs):
    return sum(forward_bytes(M, N, K) for _, K, N, M in probs)


def step_tokens(probs):
    return sum(M for _, _, _, M in probs)


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


def file_sha256(path):
    import hashlib
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


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

    def __enter__(self):
        return self.start()

    def __exit__(self, *exc):
        self.stop()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml unavailable"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "source": "nvml", "window": self.window}


# --------------------------------------------------------------- CPU oracle

def time_oracle(probs, budget_s, max_steps=None, per_problem=False, threads=1):
    """Run the CPU oracle over the workload: whole steps (or single problems,
    cycling, when per_problem) until budget_s is spent, its integer matmul on
    `threads` threads.  Returns (bytes, seconds, units, threads in effect)."""
    import oracle
    from ternary_quantized_linear_b200 import workloads
    threads = oracle.set_threads(threads)
    case = workloads.CASE_BY_NAME[WORKLOAD]
    prepared = []
    wcache = {}
    for si, K, N, M in probs:
        if si not in wcache:
            W = workloads.weights(case, si)
            s_w, _ = oracle.weight_scale(W)
            W_p, _ = oracle.quantize_pack(W, s_w)
            wcache[si] = (W_p, s_w)
        prepared.append((workloads.activations(case, si, M), wcache[si], K, N, M))
    total_b, total_s, units = 0, 0.0, 0
    t_start = time.perf_counter()
    i = 0
    while True:
        batch = [prepared[i % len(prepared)]] if per_problem else prepared
        t0 = time.perf_counter()
        for x, (W_p, s_w), K, N, M in batch:
            oracle.linear_forward(x, None, workloads.DEFAULT_EPS, W_p, s_w, K)
            total_b += forward_bytes(M, N, K)
        total_s += time.perf_counter() - t0
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
    case, probs = problems()
    # warm-up steps (untimed), then exactly `steps` timed steps; one step here is
    # one problem of the workload (cycling through the nine), so the run stays short
    time_oracle(probs, 0, max_steps=max(args.warmup, 0) or 1, per_problem=True)
    b, s, units, threads = time_oracle(probs, 0, max_steps=args.steps, per_problem=True)
    gbs = b / s / 1e9
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * s / units, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": WORKLOAD + ": " + case.description, "x_dtype": "bf16",
                   "y_dtype": "bf16"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{units} single-problem steps cycling through the nine "
                                   "decode problems, plain C oracle, 1 thread"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------- GPU path

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
    case, probs = problems()
    R = args.rotations
    eps = workloads.DEFAULT_EPS

    # ---- inputs resident in HBM: R rotation sets x 9 problems
    packed = {}
    for si in range(len(case.shapes)):
        W = torch.from_numpy(workloads.weights(case, si)).to(device)
        packed[si] = tql.bitnet_quantize_pack_weights(W)
        del W
    sets = []
    for r in range(R):
        entries = []
        for si, K, N, M in probs:
            W_p, s_w = packed[si]
            xh = workloads.activations(case, si, M)
            x = torch.from_numpy(xh.view(np.int16).copy()).view(torch.bfloat16).to(device)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            ws = torch.zeros(tql.bitnet_linear_forward_workspace_bytes(M, N, K),
                             dtype=torch.uint8, device=device)
            entries.append({"x": x, "W_p": W_p.clone(), "s_w": s_w, "y": y, "ws": ws,
                            "M": M, "N": N, "K": K})
        sets.append(entries)
    torch.cuda.synchronize()
    weight_mb_per_set = sum(e["W_p"].numel() for e in sets[0]) / 1e6

    stream = torch.cuda.Stream(device=device)
    P = ctypes.c_void_p

    # one grouped-forward description (and workspace) per rotation set
    groups = []
    for r in range(R):
        items = [(e["x"], None, eps, e["W_p"], e["s_w"], e["y"]) for e in sets[r]]
        arr, count = tql.grouped_problems(items)
        nb = tql.bitnet_linear_forward_grouped_workspace_bytes(arr, count)
        ws = torch.empty(nb, dtype=torch.uint8, device=device)
        groups.append((arr, count, ws))

    def grouped(r, sp, phases=tql.BITNET_PHASE_ALL):
        arr, count, ws = groups[r]
        rc = lib.bitnet_linear_forward_grouped(count, ctypes.cast(arr, P), P(ws.data_ptr()),
                                               ws.numel(), phases, sp)
        if rc != 0:
            raise RuntimeError(f"bitnet_linear_forward_grouped: {tql.bitnet_status_string(rc)}")

    # ---- CUDA graphs: one per rotation set (one step = one grouped call = 2
    # launches) and one holding the R steps of a whole rotation back to back,
    # so the timed loop pays one graph launch per R steps
    graphs = []
    with torch.cuda.stream(stream):
        grouped(0, P(stream.cuda_stream))  # first call sets up the device state
        stream.synchronize()
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                grouped(r, P(torch.cuda.current_stream().cuda_stream))
            graphs.append(g)
        rotation = torch.cuda.CUDAGraph()
        with torch.cuda.graph(rotation, stream=stream):
            for r in range(R):
                grouped(r, P(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()

    def run_steps(k):
        # exactly k steps, cycling through the rotation sets
        for _ in range(k // R):
            rotation.replay()
        for r in range(k % R):
            graphs[r].replay()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local_rank])

    # ---- warm-up, then exactly K timed steps (graph replays).  The clock
    # sampler runs from the warm-up through the kernel-timing replays below:
    # the timed steps alone last a few milliseconds, about one NVML sample.
    clocks = ClockSampler(local_rank, window="warm-up, the timed steps and the kernel-timing "
                                              "graph replays (all back-to-back GPU work)")
    clocks.start()
    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        run_steps(args.steps)
        e1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    barrier()
    local_ms = e0.elapsed_time(e1)
    max_ms = max_over_ranks(local_ms, world, device)
    sb = step_bytes(probs)
    value = job_throughput(sb, args.steps, world, max_ms)
    ms_per_step = max_ms / args.steps
    launches = 2 * args.steps

    # ---- kernel durations with CUDA events: the grouped matmul (dominant
    # kernel) and the grouped activation quant, each captured alone as CUDA
    # graphs over the rotation sets (the matmul phase reads the activations
    # the full steps above left in each set's workspace) and replayed
    # back to back: the average launch duration in a steady stream.
    def phase_ms(phases):
        gs = []
        with torch.cuda.stream(stream):
            for r in range(R):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    grouped(r, P(torch.cuda.current_stream().cuda_stream), phases)
                gs.append(g)
            for i in range(args.warmup):
                gs[i % R].replay()
            stream.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(args.steps):
                gs[i % R].replay()
            b.record(stream)
            stream.synchronize()
        ms = a.elapsed_time(b) / args.steps
        del gs
        return ms

    m_avg = phase_ms(tql.BITNET_PHASE_MATMUL)
    q_avg = phase_ms(tql.BITNET_PHASE_QUANTIZE)
    clocks.stop()
    gemv_b = sum(gemv_bytes(M, N, K) for _, K, N, M in probs)
    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = gemv_b / (m_avg * 1e-3) / 1e9
    sha = file_sha256(os.path.join(ROOT, "ternary_quantized_linear_b200", "csrc", "gemv.cuh"))
    traffic = GEMV_TRAFFIC["bytes_per_launch"] if GEMV_TRAFFIC["src_sha256"] == sha else None

    # ---- the same nine problems one launch pair at a time (two-phase single API)
    single = []
    one = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in probs]
    acc_q = {j: [] for j in range(len(probs))}
    acc_m = {j: [] for j in range(len(probs))}
    with torch.cuda.stream(stream):
        for i in range(min(args.steps, 20) + 2):
            r = i % R
            torch.cuda._sleep(2_000_000)
            for j, e in enumerate(sets[r]):
                one[j][0].record(stream)
                tql.bitnet_linear_quantize_input(e["x"], None, eps, e["N"], e["ws"],
                                                 stream=stream)
                one[j][1].record(stream)
                tql.bitnet_linear_matmul(e["W_p"], e["s_w"], e["M"], e["K"], e["ws"], y=e["y"],
                                         stream=stream)
                one[j][2].record(stream)
            stream.synchronize()
            if i >= 2:
                for j in range(len(probs)):
                    acc_q[j].append(one[j][0].elapsed_time(one[j][1]))
                    acc_m[j].append(one[j][1].elapsed_time(one[j][2]))
    for j, (si, K, N, M) in enumerate(probs):
        t = statistics.mean(acc_m[j])
        single.append({"K": K, "N": N, "M": M, "matmul_us": round(1e3 * t, 2),
                       "matmul_gbs": round(gemv_bytes(M, N, K) / (t * 1e-3) / 1e9, 1),
                       "quant_us": round(1e3 * statistics.mean(acc_q[j]), 2)})

    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                "kernel": "ternary_gemv_kernel, one grouped launch over the nine problems "
                          "(matmul + fused dequant)",
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                "algorithmic_bytes_per_launch": gemv_b,
                "avg_launch_us": round(1e3 * m_avg, 2),
                "quant_kernel_us": round(1e3 * q_avg, 2),
                "how": "CUDA events around back-to-back CUDA-graph replays of the matmul "
                       "phase alone (6 rotating weight sets), average per launch",
                "single_problem_launches": single}

    # ---- end to end through the public call with host buffers: each set's
    # nine inputs live in one pinned host buffer and one device buffer (and
    # likewise the outputs), so a step is one upload, one grouped call and
    # one download.
    e2e = None
    if not args.no_e2e:
        def packed(shapes, dtype):
            # 128-byte aligned offsets of each tensor in one flat buffer
            offs, n = [], 0
            for shp in shapes:
                offs.append(n)
                n += -(-shp[0] * shp[1] // 64) * 64
            return offs, n

        e2e_sets, e2e_yoffs = [], []
        for r in range(R):
            xs = [tuple(e["x"].shape) for e in sets[r]]
            ys = [tuple(e["y"].shape) for e in sets[r]]
            xo, xn = packed(xs, torch.bfloat16)
            yo, yn = packed(ys, torch.bfloat16)
            dx = torch.empty(xn, dtype=torch.bfloat16, device=device)
            dy = torch.empty(yn, dtype=torch.bfloat16, device=device)
            hx = torch.empty(xn, dtype=torch.bfloat16).pin_memory()
            hy = torch.empty(yn, dtype=torch.bfloat16).pin_memory()
            items = []
            for j, e in enumerate(sets[r]):
                xv = dx[xo[j]:xo[j] + xs[j][0] * xs[j][1]].view(xs[j])
                hx[xo[j]:xo[j] + xs[j][0] * xs[j][1]].view(xs[j]).copy_(e["x"].cpu())
                yv = dy[yo[j]:yo[j] + ys[j][0] * ys[j][1]].view(ys[j])
                items.append((xv, None, eps, e["W_p"], e["s_w"], yv))
            arr, count = tql.grouped_problems(items)
            nb = tql.bitnet_linear_forward_grouped_workspace_bytes(arr, count)
            ws = torch.empty(nb, dtype=torch.uint8, device=device)
            e2e_sets.append((dx, dy, hx, hy, arr, count, ws, items))
            e2e_yoffs.append(yo)
        h2d = sum(e["x"].numel() * 2 for e in sets[0])
        d2h = sum(e["y"].numel() * 2 for e in sets[0])
        def grouped_call(r, st):
            _, _, _, _, arr, count, ws, _ = e2e_sets[r]
            rc = lib.bitnet_linear_forward_grouped(count, ctypes.cast(arr, P), P(ws.data_ptr()),
                                                   ws.numel(), tql.BITNET_PHASE_ALL,
                                                   P(st.cuda_stream))
            if rc != 0:
                raise RuntimeError(tql.bitnet_status_string(rc))

        def e2e_serial():
            # one stream: upload, call, download, step after step
            def step(r):
                dx, dy, hx, hy = e2e_sets[r][:4]
                dx.copy_(hx, non_blocking=True)
                grouped_call(r, stream)
                hy.copy_(dy, non_blocking=True)

            with torch.cuda.stream(stream):
                for i in range(args.warmup):
                    step(i % R)
                stream.synchronize()
                barrier()
                a0 = torch.cuda.Event(enable_timing=True)
                a1 = torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                for i in range(args.steps):
                    step(i % R)
                a1.record(stream)
                stream.synchronize()
            return a0.elapsed_time(a1)

        def e2e_pipelined():
            # Three streams -- uploads, grouped calls, downloads -- so step i's
            # upload overlaps step i-1's call and download.  Per rotation set,
            # events order upload -> call -> download and gate the reuse of
            # its buffers: an upload waits for the set's previous call (its
            # input buffer is free), a call for the set's previous download
            # (its output buffer is free).  The copies and event operations go
            # straight to the CUDA driver (handles and pointers resolved before
            # the loop) so the host keeps ahead of the device.
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
            for r in range(R):
                dx, dy, hx, hy, arr, count, ws, _ = e2e_sets[r]
                nx, ny = dx.numel() * dx.element_size(), dy.numel() * dy.element_size()
                assert nx == hx.numel() * hx.element_size() and hx.is_pinned()
                assert ny == hy.numel() * hy.element_size() and hy.is_pinned()
                plan.append((U64(dx.data_ptr()), VP(hx.data_ptr()), SZ(nx),
                             VP(hy.data_ptr()), U64(dy.data_ptr()), SZ(ny),
                             count, ctypes.cast(arr, P), P(ws.data_ptr()), ws.numel()))
            call = lib.bitnet_linear_forward_grouped
            phase = tql.BITNET_PHASE_ALL

            def step(r):
                dxp, hxp, nx, hyp, dyp, ny, count, arr_p, ws_p, nb = plan[r]
                if used[r]:
                    ok(wait_ev(h_up, called[r], 0), "cuStreamWaitEvent")
                ok(h2d_copy(dxp, hxp, nx, h_up), "cuMemcpyHtoDAsync")
                ok(ev_record(up[r], h_up), "cuEventRecord")
                ok(wait_ev(h_c, up[r], 0), "cuStreamWaitEvent")
                if used[r]:
                    ok(wait_ev(h_c, down[r], 0), "cuStreamWaitEvent")
                rc = call(count, arr_p, ws_p, nb, phase, h_c)
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

            try:
                for i in range(args.warmup):
                    step(i % R)
                join()
                torch.cuda.synchronize()
                barrier()
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
            finally:
                torch.cuda.synchronize()
                for e in events:
                    ev_destroy(e)
            # the downloads hold what the device path computed for each set
            for r in range(R):
                if not used[r]:
                    continue
                hy, items = e2e_sets[r][3], e2e_sets[r][7]
                got = torch.cat([hy[o:o + it[5].numel()] for o, it in zip(e2e_yoffs[r], items)])
                want = torch.cat([e["y"].reshape(-1).cpu() for e in sets[r]])
                if not torch.equal(got.view(torch.int16), want.view(torch.int16)):
                    raise RuntimeError(f"pipelined end-to-end outputs of set {r} differ")
            return a0.elapsed_time(a1)

        how_serial = ("per step: one pinned-host -> device copy of the nine inputs, one "
                      "bitnet_linear_forward_grouped call (C ABI, eager), one device -> "
                      "pinned-host copy of the nine outputs, all on one stream; device-timed")
        how_pipe = ("per step: one pinned-host -> device copy of the nine inputs, one "
                    "bitnet_linear_forward_grouped call (C ABI, eager), one device -> "
                    "pinned-host copy of the nine outputs; uploads, calls and downloads on "
                    "three streams ordered per rotation set by events (copies and events "
                    "issued through the CUDA driver API), so step i's upload overlaps step "
                    "i-1's call and download; every step's copies inside the timed region; "
                    "outputs checked against the device path; device-timed")
        note = None
        try:
            local = e2e_pipelined()
            how = how_pipe
        except Exception as exc:  # noqa: BLE001 -- any failure: measure on one stream
            torch.cuda.synchronize()
            note = f"pipelined measurement failed ({exc}); serial measurement instead"
            local = e2e_serial()
            how = how_serial
        e2e_ms = max_over_ranks(local, world, device)
        e2e = {"value": job_throughput(sb, args.steps, world, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / args.steps, "how": how}
        if note:
            e2e["note"] = note

    # ---- prefill extra: tcgen05 GEMM TOPS on the Llama-3-8B FFN shapes
    prefill = None
    if not args.no_prefill:
        prefill = measure_prefill(args, device, stream, peaks, peak_src)

    # ---- offline weight quant + pack, timed on its own (not in the metric)
    weight_pack = None
    if not args.no_weight_pack:
        try:
            weight_pack = measure_weight_pack(args, device, stream, hbm_peak)
        except Exception as exc:  # noqa: BLE001 -- report, keep the line
            weight_pack = {"error": str(exc)}

    # ---- CPU baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        b, s, units, threads = time_oracle(probs, args.cpu_budget)
        cpu = {"value": b / s / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{units} full decode step(s) (all nine problems) of the plain C "
                         f"oracle, {threads} thread(s), {s:.1f} s"}
        # the same oracle with its integer matmul spread over every host core
        ncores = os.cpu_count() or 1
        b, s, units, threads = time_oracle(probs, args.cpu_budget / 2, threads=ncores)
        cpu["all_cores"] = {"value": b / s / 1e9, "unit": "GB/s", "cores": threads,
                            "sample": f"{units} full decode step(s), integer matmul on "
                                      f"{threads} thread(s), {s:.1f} s"}

    if world > 1:
        import torch.distributed as dist
        for g in graphs:
            del g
        graphs.clear()
        del rotation
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic",
            "config": {"workload": WORKLOAD + ": " + case.description,
                       "problems": [[K, N, M] for _, K, N, M in probs],
                       "x_dtype": "bf16", "y_dtype": "bf16",
                       "l2": f"inputs larger than L2: {R} rotating weight/activation sets, "
                             f"{R * weight_mb_per_set:.0f} MB of packed weights",
                       "launch": "one bitnet_linear_forward_grouped call per step (a grouped "
                                 "activation-quant launch + a grouped matmul launch with "
                                 "programmatic dependent launch); the R rotation steps "
                                 "captured back to back in one CUDA graph, replayed "
                                 "steps/R times (single-step graphs for a remainder)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "tok_s": round(world * step_tokens(probs) * args.steps / (max_ms * 1e-3), 1),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks.summary(),
            "prefill": prefill,
            "weight_pack": weight_pack,
        }
        print(json.dumps(line), flush=True)
    return 0


def measure_weight_pack(args, device, stream, hbm_peak):
    """bitnet_quantize_pack_weights on the decode workload's three fp32
    matrices (261 MB together, more than L2), cycled, outputs preallocated:
    the absmean pass reads W, the quantize pass reads it again and writes the
    packed codes (the scale must be known before any code is decided)."""
    import torch

    import ternary_quantized_linear_b200 as tql
    from ternary_quantized_linear_b200 import workloads

    case = workloads.CASE_BY_NAME[WORKLOAD]
    mats = []
    for si, (K, N) in enumerate(case.shapes):
        W = torch.from_numpy(workloads.weights(case, si)).to(device)
        W_p = torch.empty((N, K // 4), dtype=torch.uint8, device=device)
        s_w = torch.empty((1,), dtype=torch.float32, device=device)
        nb = max(tql.bitnet_quantize_pack_weights_workspace_bytes(N, K), 256)
        ws = torch.empty(nb, dtype=torch.uint8, device=device)
        mats.append((W, W_p, s_w, ws, N, K))
    n = len(mats)
    reps = max(3, min(args.steps, 30))
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3) * n):
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
        ms = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(j, reps * n, n)) / reps
        b = 2 * 4 * N * K + N * K // 4
        tot_b += b
        tot_ms += ms
        per.append({"N": N, "K": K, "us": round(1e3 * ms, 2),
                    "gbs": round(b / (ms * 1e-3) / 1e9, 1)})
    gbs = tot_b / (tot_ms * 1e-3) / 1e9
    return {"workload": f"{WORKLOAD} weights, fp32, cycled", "matrices": per,
            "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / hbm_peak, 4),
            "bytes": "two reads of W (absmean, then quantize) + the packed write",
            "how": "CUDA events around each call on the launching stream, "
                   f"{reps} calls per matrix after warm-up"}


def measure_prefill(args, device, stream, peaks, peak_src):
    """Tensor-core path on the Llama-3-8B FFN shapes at M = 2048 (not the
    headline number): TOPS of the GEMM kernel alone and of the whole forward."""
    import numpy as np
    import torch

    import ternary_quantized_linear_b200 as tql
    from ternary_quantized_linear_b200 import workloads

    case = workloads.CASE_BY_NAME["prefill_llama3_8b"]
    M = 2048
    out = []
    i8_peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    for si, (K, N) in enumerate(case.shapes):
        W = torch.from_numpy(workloads.weights(case, si)).to(device)
        W_p, s_w = tql.bitnet_quantize_pack_weights(W)
        del W
        xh = workloads.activations(case, si, M)
        R = 6
        xs = [torch.from_numpy(xh.view(np.int16).copy()).view(torch.bfloat16).to(device)
              for _ in range(R)]
        wps = [W_p.clone() for _ in range(R)]
        y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ws = torch.zeros(tql.bitnet_linear_forward_workspace_bytes(M, N, K), dtype=torch.uint8,
                         device=device)
        iters = 20
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(iters)]
        with torch.cuda.stream(stream):
            for i in range(3):
                tql.bitnet_linear_forward(xs[i % R], None, 1e-5, wps[i % R], s_w, y=y,
                                          workspace=ws, stream=stream)
            for i in range(iters):
                evs[i][0].record(stream)
                tql.bitnet_linear_quantize_input(xs[i % R], None, 1e-5, N, ws, stream=stream)
                evs[i][1].record(stream)
                tql.bitnet_linear_matmul(wps[i % R], s_w, M, K, ws, y=y, stream=stream)
                evs[i][2].record(stream)
            stream.synchronize()
        gemm_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
        fwd_ms = statistics.median(e[0].elapsed_time(e[2]) for e in evs)
        ops = 2.0 * M * N * K
        out.append({"K": K, "N": N, "M": M, "gemm_us": round(1e3 * gemm_ms, 2),
                    "gemm_tops": round(ops / (gemm_ms * 1e-3) / 1e12, 1),
                    "forward_tops": round(ops / (fwd_ms * 1e-3) / 1e12, 1)})
    tops = [o["gemm_tops"] for o in out]
    return {"workload": "prefill_llama3_8b at M=2048 (K=4096->N=14336, K=14336->N=4096)",
            "shapes": out, "gemm_tops_mean": round(statistics.mean(tops), 1),
            "frac_of_int8_peak": round(statistics.mean(tops) / i8_peak, 4),
            "int8_peak_tops": i8_peak,
            "int8_peak_source": f"{peak_src} bf16 burst x 2 (dense int8 = 2x bf16 rate)",
            "frac_of_4500_tops_spec": round(statistics.mean(tops) / 4500.0, 4)}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--rotations", type=int, default=6)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-weight-pack", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
