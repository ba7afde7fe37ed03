#!/usr/bin/env python
"""Throughput of the NVFP4 quantize / fake-quant hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step is one pass of the whole path over one batch: the activation observer
(global amax + EMA update; with N > 1 ranks the amax is MAX-all-reduced over NCCL
first, as a data-parallel QAT step does), fake-quant with the observed amax, quantize
to packed E2M1 codes + E4M3 scales, and dequantize back to bf16.  Every rank owns its
own bf16 [65536, 8192] activation (1 GiB, N(0,1)), so the work per GPU is fixed
(weak scaling).  ``value`` is the algorithmic bytes of all ranks' steps divided by the
slowest rank's device time, in GB/s.

Rank 0 prints one JSON line.  The native arm also reports the dominant kernel's
roofline, the CPU oracle's throughput on a bounded sample (cpu_baseline), an
end-to-end figure with host buffers (e2e), the SM clocks seen during the timed region
and the number of library kernels launched.  ``--impl reference`` times the CPU oracle
instead (the reference arm), on a bounded sample of the same workload.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 fake-quant/quantize GB/s and fraction of B200 HBM roofline"
UNIT = "GB/s"
# Algorithmic (minimal) bytes per element of each kernel of the step.
KERNEL_BYTES = {"amax": 2.0, "fake_quant": 4.0, "quantize": 2.0 + 0.5 + 1.0 / 16, "dequantize": 0.5 + 1.0 / 16 + 2.0}
STEP_BYTES = sum(KERNEL_BYTES.values())  # 11.125 bytes per element
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CSRC = os.path.join(ROOT, "qat_nvfp4_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--rows", type=int, default=65536)
    p.add_argument("--cols", type=int, default=8192)
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--cpu-rows", type=int, default=2048, help="rows of the oracle sample (cpu_baseline)")
    p.add_argument("--skip-e2e", action="store_true")
    p.add_argument("--e2e-serial", action="store_true",
                   help="e2e on one stream (upload, step, download in turn) instead of the two-buffer "
                        "pipeline that overlaps a step's download with the next step's upload")
    p.add_argument("--skip-cpu-baseline", action="store_true")
    p.add_argument("--sweep", metavar="OUT_JSON", default=None,
                   help="instead of the one-line step benchmark, time each kernel on every workload size "
                        "(L2 flushed before each rep), print a table and write it as JSON to OUT_JSON")
    p.add_argument("--linear", metavar="OUT_JSON", default=None,
                   help="instead of the step benchmark, time the W4A16 linear (x . W^T with W stored as NVFP4 "
                        "records) for several token counts on the pages' weight shapes, beside dequantize + "
                        "torch bf16 linear and a bf16 linear on an unquantized weight; print a table, write JSON")
    p.add_argument("--strided", metavar="OUT_JSON", default=None,
                   help="time amax / quantize / in-place fake-quant on the q, k and v column views of a fused "
                        "[16384, 6144] projection output against the same calls on contiguous copies "
                        "(L2 flushed before each rep), print a table and write it as JSON to OUT_JSON")
    p.add_argument("--linear-shape", metavar="M,K,N", default=None,
                   help="run the W4A16 linear three times on one shape (tokens M, in-features K, out-features "
                        "N; N(0, 1) activations, N(0, 0.02) weight) and exit: the command profiled by ncu")
    return p.parse_args()


def workload_config(args, world):
    return {
        "workload": f"bf16 activation {args.rows}x{args.cols} ~ N(0,1) per GPU; step = EMA(0.01) observer amax"
                    f"{' + NCCL MAX all-reduce' if world > 1 else ''} -> fake-quant -> quantize -> dequantize",
        "shape": [args.rows, args.cols],
        "bytes_per_elem_per_step": STEP_BYTES,
        "l2": "inputs larger than L2 (1 GiB per GPU vs 126 MB), no flush" if args.rows * args.cols * 2 > (256 << 20)
              else "inputs smaller than 2x L2: L2-warm figures",
        "parallelism": f"dp{world}",
    }


# The sources of the kernels the step runs (the W4A16 linear has its own file).
STEP_SOURCES = ("nvfp4_device.cuh", "nvfp4_runtime.h", "nvfp4_stream.cuh", "nvfp4_reduce.cuh", "nvfp4_encode.cuh",
                "nvfp4_ragged.cuh", "nvfp4_strided.cuh", "nvfp4_kernels.cu")


def source_digest():
    h = hashlib.sha256()
    for fn in STEP_SOURCES:
        with open(os.path.join(CSRC, fn), "rb") as f:
            h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()


def bf16_peak():
    """Measured dense bf16 tensor throughput (TFLOP/s), burst figure: the linear kernels are
    timed one launch at a time."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst cuBLAS GEMM)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback (earlier measurement on this pool)"


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, burst copy)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback (earlier measurement on this pool)"


def stored_traffic(kernel, numel):
    """dram bytes per launch from the committed ncu summary, scaled to `numel` elements,
    or None if there is none or the kernel sources changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if t.get("source_sha256") != source_digest():
        return None
    return t["dram_bytes_per_elem"] * numel


# ---------------------------------------------------------------------------------------
# Clocks during the timed region (NVML, polled from a thread).

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index, period_s=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - report, never fail the bench on telemetry
            self.nvml, self.error = None, str(e)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
            mask = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            self.reasons |= {n for n, b in self.REASONS.items() if mask & b}
        except Exception:  # noqa: BLE001
            pass

    def start(self):
        if self.nvml:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self.nvml and self._thread:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if not self.nvml:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# The CPU oracle step (cpu_baseline and the reference arm).

def oracle_step(x_bits, state=-1.0):
    import oracle
    a = oracle.amax(x_bits)
    s = oracle.observer_update(state, a, oracle.EMA, 0.01)
    oracle.fake_quant(x_bits, s)
    gs = oracle.global_scale(s)
    packed, scales = oracle.quantize(x_bits, gs)
    oracle.dequantize(packed, scales, gs, *x_bits.shape)
    return s


def time_oracle(x_bits, repeats=1):
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle_step(x_bits)
    return (time.perf_counter() - t0) / repeats


def time_oracle_all_cores(x_bits, threads):
    """The same oracle step with each phase run over row ranges on `threads` threads (the
    oracle's C calls release the GIL; rows are independent in every per-block step, and
    the amax of the sample is the max of the ranges' amaxes).  Returns seconds."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    M, N = x_bits.shape
    step = -(-M // threads)
    ranges = [(r, min(M, r + step)) for r in range(0, M, step)]
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as pool:
        a = max(pool.map(lambda rr: oracle.amax(x_bits[rr[0]:rr[1]]), ranges))
        s = oracle.observer_update(-1.0, a, oracle.EMA, 0.01)
        list(pool.map(lambda rr: oracle.fake_quant(x_bits[rr[0]:rr[1]], s), ranges))
        gs = oracle.global_scale(s)

        def q_dq(rr):
            part = x_bits[rr[0]:rr[1]]
            packed, scales = oracle.quantize(part, gs)
            oracle.dequantize(packed, scales, gs, *part.shape)
        list(pool.map(q_dq, ranges))
    return time.perf_counter() - t0


# ---------------------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from qat_nvfp4_b200 import synthetic
    cols = args.cols
    # size the sample so that warm-up + steps end in about two minutes
    probe = synthetic.activation_normal((16, cols), seed=12)
    per_row = time_oracle(probe) / 16
    budget = 120.0 / max(1, args.steps + args.warmup)
    rows = int(max(8, min(args.rows, budget / per_row)))
    x = synthetic.activation_normal((rows, cols), seed=12)
    for _ in range(args.warmup):
        oracle_step(x)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(x)
    elapsed = time.perf_counter() - t0
    value = STEP_BYTES * rows * cols * args.steps / elapsed / 1e9
    sample = (f"first {rows} of {args.rows} rows x {cols} (one oracle step per timed step: amax, EMA observer, "
              f"fake-quant, quantize, dequantize), single thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_native(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from qat_nvfp4_b200 import nvfp4 as nv
    from qat_nvfp4_b200 import synthetic

    M, N = args.rows, args.cols
    numel = M * N
    x = synthetic.activation_normal_device((M, N), seed=5 + 7 + 1000 * rank, device=dev)
    y = torch.empty_like(x)
    y2 = torch.empty_like(x)
    B = (N + 15) // 16  # blocks per row (rows are zero-padded to 16 * B columns)
    packed = torch.empty((M, 8 * B), dtype=torch.uint8, device=dev)
    scales = torch.empty((M, B), dtype=torch.uint8, device=dev)
    gs = torch.empty(1, dtype=torch.float32, device=dev)
    cur = torch.empty(1, dtype=torch.float32, device=dev)
    state = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
    ws = nv.new_workspace(dev)
    stream = torch.cuda.current_stream(dev)

    stages = ["amax", "fake_quant", "quantize", "dequantize"]

    def step_on(xb, yb, y2b, pb, sb, gb, ev=None, st=None):
        """One step on the given buffers (the observer state is shared: steps run in order)."""
        def mark(i):
            if ev is not None:
                ev[i].record(st if st is not None else stream)
        mark(0)
        if world == 1:
            nv.nvfp4_observe_amax(xb, state, kind="minmax", decay=0.01, cur_out=cur, workspace=ws)
        else:
            nv.nvfp4_amax(xb, out=cur, workspace=ws)
            dist.all_reduce(cur, op=dist.ReduceOp.MAX)
            nv.nvfp4_observer_update(state, cur, kind="minmax", decay=0.01)
        mark(1)
        nv.nvfp4_fake_quant(xb, state, out=yb)
        mark(2)
        nv.nvfp4_quantize(xb, state, pb, sb, gb)
        mark(3)
        nv.nvfp4_dequantize(pb, sb, gb, out=y2b, n_cols=N)
        mark(4)

    def step(ev=None):
        step_on(x, y, y2, packed, scales, gs, ev)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    def max_over_ranks(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return t.item()

    for _ in range(max(args.warmup, 3)):
        step()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier()
    launches0 = nv.nvfp4_kernel_launch_count()
    sampler.start()
    start.record(stream)
    for k in range(args.steps):
        step(events[k])
    end.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    launches = nv.nvfp4_kernel_launch_count() - launches0
    barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(end))
    stage_ms = {s: statistics.fmean(events[k][i].elapsed_time(events[k][i + 1]) for k in range(args.steps))
                for i, s in enumerate(stages)}
    stage_ms = {s: max_over_ranks(v) for s, v in stage_ms.items()}

    value = world * args.steps * numel * STEP_BYTES / (elapsed_ms / 1e3) / 1e9
    peak, peak_src = hbm_peak()
    kernels = {s: {"ms": stage_ms[s], "GB/s": numel * KERNEL_BYTES[s] / (stage_ms[s] / 1e3) / 1e9,
                   "bytes_per_elem": KERNEL_BYTES[s]} for s in stages}
    for s in stages:
        kernels[s]["frac_of_hbm_peak"] = kernels[s]["GB/s"] / peak
    fq = kernels["fake_quant"]
    roofline = {"bound": "hbm", "kernel": "fake_quant_kernel", "achieved": fq["GB/s"], "peak": peak,
                "unit": "GB/s", "frac": fq["GB/s"] / peak, "traffic": stored_traffic("fake_quant", numel),
                "algorithmic_bytes_per_launch": numel * KERNEL_BYTES["fake_quant"], "peak_source": peak_src}

    # ---- end to end with host buffers: H2D of x, the step, D2H of every output ----
    e2e = None
    if not args.skip_e2e and args.e2e_serial:
        x_h = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
        x_h.copy_(x)
        outs = [(y, torch.empty_like(y, device="cpu", pin_memory=True)),
                (y2, torch.empty_like(y2, device="cpu", pin_memory=True)),
                (packed, torch.empty_like(packed, device="cpu", pin_memory=True)),
                (scales, torch.empty_like(scales, device="cpu", pin_memory=True)),
                (gs, torch.empty_like(gs, device="cpu", pin_memory=True)),
                (state, torch.empty_like(state, device="cpu", pin_memory=True))]

        def e2e_step():
            x.copy_(x_h, non_blocking=True)
            step()
            for d, h in outs:
                h.copy_(d, non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    elif not args.skip_e2e:
        # Two buffer sets; step k uses set k % 2 on three streams (upload, compute, download),
        # so step k's download overlaps step k + 1's upload (PCIe is full duplex).  Every step
        # still uploads its x from pinned memory and downloads all of its outputs inside the
        # timed region; the observer state is snapshotted per set at the end of each step.
        x_h = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
        x_h.copy_(x)
        sets = []
        for b in range(2):
            bufs = (x, y, y2, packed, scales, gs) if b == 0 else tuple(torch.empty_like(t) for t in
                                                                       (x, y, y2, packed, scales, gs))
            snap = torch.empty_like(state)
            outs = [(d, torch.empty_like(d, device="cpu", pin_memory=True)) for d in bufs[1:] + (snap,)]
            sets.append((bufs, snap, outs))
        s_up, s_comp, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        up_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        down_done = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(k):
            b = k % 2
            bufs, snap, outs = sets[b]
            with torch.cuda.stream(s_up):
                if k >= 2:
                    s_up.wait_event(comp_done[b])  # step k - 2 has read this x
                bufs[0].copy_(x_h, non_blocking=True)
                up_done[b].record(s_up)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(up_done[b])
                if k >= 2:
                    s_comp.wait_event(down_done[b])  # step k - 2's outputs have been read out
                step_on(*bufs)
                snap.copy_(state)
                comp_done[b].record(s_comp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(comp_done[b])
                for d, h in outs:
                    h.copy_(d, non_blocking=True)
                down_done[b].record(s_down)

        for k in range(2):
            e2e_step(k)
        torch.cuda.synchronize(dev)
        barrier()
        outs = sets[0][2]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_up)
        for k in range(args.e2e_steps):
            e2e_step(k)
        s_down.wait_stream(s_up)
        s_down.wait_stream(s_comp)
        e1.record(s_down)
        torch.cuda.synchronize(dev)
    if not args.skip_e2e:
        e2e_ms = max_over_ranks(e0.elapsed_time(e1))
        d2h = sum(d.numel() * d.element_size() for d, _ in outs)
        e2e = {"value": world * args.e2e_steps * numel * STEP_BYTES / (e2e_ms / 1e3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": numel * 2, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "ms_per_step": e2e_ms / args.e2e_steps,
               "schedule": "serial (one stream)" if args.e2e_serial else
               "two buffer sets, upload / compute / download streams: a step's download overlaps the next upload"}

    # ---- the CPU oracle on a bounded sample (rank 0, one GPU only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        import oracle
        oracle.amax(x[:1].contiguous().view(torch.int16).cpu().numpy().view("uint16"))  # load before threads
        rows = min(args.cpu_rows, M)
        sample = x[:rows].contiguous().view(torch.int16).cpu().numpy().view("uint16")
        t1 = time_oracle(sample)
        cores = len(os.sched_getaffinity(0))
        rows_all = min(M, args.cpu_rows * max(1, cores // 2))
        sample_all = x[:rows_all].contiguous().view(torch.int16).cpu().numpy().view("uint16")
        tn = time_oracle_all_cores(sample_all, cores)
        cpu = {"value": STEP_BYTES * rows_all * N / tn / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"first {rows_all} of {M} rows x {N}: one oracle step (amax, EMA observer, fake-quant, "
                         f"quantize, dequantize), each phase over row ranges on {cores} threads, {tn:.1f} s",
               "single_thread": {"value": STEP_BYTES * rows * N / t1 / 1e9, "unit": UNIT, "cores": 1,
                                 "sample": f"first {rows} rows, one thread, {t1:.1f} s"}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(args, world), "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": sampler.summary(), "kernels": kernels,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def run_sweep(args):
    """Per-kernel GB/s on every workload shape: the activation size sweep 1024^2 .. 65536x8192,
    the 256x1024 and 4096x4096 weights, the 8192x4096 activations and 14336x4096 weight,
    and the q/k/v siblings.  Each rep is preceded by a read of a 512 MB buffer, so no input
    starts in L2 and no dirty line is left behind; CUDA events, median of the reps."""
    import torch
    from qat_nvfp4_b200 import nvfp4 as nv
    from qat_nvfp4_b200 import synthetic

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_src = hbm_peak()
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)
    ws = nv.new_workspace(dev)
    reps = 15

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.sum(dtype=torch.int32)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        return sorted(ts)[len(ts) // 2] / 1e3

    shapes = [("activation sweep", s) for s in synthetic.SWEEP_SHAPES]
    shapes += [("grid-block weight", (256, 1024)), ("outlier weight", (4096, 4096)),
               ("W4A4 activation", (8192, 4096)), ("MLP weight", (14336, 4096))]
    rows = []
    for name, (M, N) in shapes:
        x = synthetic.activation_normal_device((M, N), 99, dev)
        n = M * N
        amax = nv.nvfp4_amax(x)
        y = torch.empty_like(x)
        packed, scales, gs = nv.nvfp4_quantize(x, amax)
        packed32, scales32, _ = nv.nvfp4_quantize(x, amax, block=32)
        packed_f, scales_f = nv.nvfp4_quantize_f32scale(x)
        scales_mma = torch.empty(nv.mma_scale_bytes(M, N), dtype=torch.uint8, device=dev)
        t = {
            "amax": (2.0, timed(lambda: nv.nvfp4_amax(x, out=amax, workspace=ws))),
            "fake_quant": (4.0, timed(lambda: nv.nvfp4_fake_quant(x, amax, out=y))),
            "fake_quant_with_own_amax": (4.0, timed(lambda: nv.nvfp4_fake_quant_fused(x, out=y, amax_out=amax,
                                                                                      workspace=ws))),
            "quantize": (2.5625, timed(lambda: nv.nvfp4_quantize(x, amax, packed, scales, gs))),
            "quantize_with_own_amax": (2.5625, timed(lambda: nv.nvfp4_quantize_fused(x, packed, scales, gs, amax,
                                                                                      workspace=ws))),
            "quantize_mma": (2.5625, timed(lambda: nv.nvfp4_quantize_mma(x, amax, packed, scales_mma, gs))),
            "dequantize": (2.5625, timed(lambda: nv.nvfp4_dequantize(packed, scales, gs, out=y))),
            # blocks of 32: 1/32 of a scale byte per element
            "fake_quant_b32": (4.0, timed(lambda: nv.nvfp4_fake_quant(x, amax, out=y, block=32))),
            "quantize_b32": (2.53125, timed(lambda: nv.nvfp4_quantize(x, amax, packed32, scales32, gs, block=32))),
            "dequantize_b32": (2.53125, timed(lambda: nv.nvfp4_dequantize(packed32, scales32, gs, out=y,
                                                                          block=32))),
            # the fp32-scale flavour: blocks of 32, a 4-byte scale per block (1/8 byte per element)
            "fake_quant_f32s": (4.0, timed(lambda: nv.nvfp4_fake_quant_f32scale(x, out=y))),
            "quantize_f32s": (2.625, timed(lambda: nv.nvfp4_quantize_f32scale(x, packed_f, scales_f))),
            "dequantize_f32s": (2.625, timed(lambda: nv.nvfp4_dequantize_f32scale(packed_f, scales_f, out=y))),
        }
        rec = {"workload": name, "shape": [M, N], "bytes": 2 * n}
        for k, (bpe, sec) in t.items():
            rec[k] = {"us": sec * 1e6, "GB/s": n * bpe / sec / 1e9, "frac": n * bpe / sec / 1e9 / peak}
        rows.append(rec)
        del x, y, packed, scales, scales_mma, packed32, scales32, packed_f, scales_f
    # the q/k/v siblings: shared amax + fake-quant of all three in one call
    qkv = [synthetic.activation_normal_device(s, 98, dev) for s in ((4096, 4096), (1024, 4096), (1024, 4096))]
    outs = [torch.empty_like(t) for t in qkv]
    n = sum(t.numel() for t in qkv)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    sec = timed(lambda: nv.nvfp4_fake_quant_siblings(qkv, outs, amax))
    rows.append({"workload": "q/k/v siblings (shared amax + fake-quant, 2 + 4 bytes/elem)", "shape": [6144, 4096],
                 "bytes": 2 * n, "siblings": {"us": sec * 1e6, "GB/s": n * 6.0 / sec / 1e9,
                                               "frac": n * 6.0 / sec / 1e9 / peak}})

    cols = ["amax", "fake_quant", "fake_quant_with_own_amax", "quantize", "quantize_with_own_amax", "quantize_mma",
            "dequantize", "fake_quant_b32", "quantize_b32", "dequantize_b32", "fake_quant_f32s", "quantize_f32s",
            "dequantize_f32s"]
    print(f"peak {peak:.1f} GB/s ({peak_src}); GB/s of algorithmic bytes (frac of peak); L2 flushed by a read")
    print("| workload | shape | " + " | ".join(cols) + " |")
    print("|---|---|" + "---|" * len(cols))
    for r in rows:
        if "siblings" in r:
            v = r["siblings"]
            print(f"| {r['workload']} | {r['shape'][0]}x{r['shape'][1]} | " + " | ".join(
                [f"{v['GB/s']:.0f} ({v['frac']:.2f})"] + [""] * (len(cols) - 1)) + " |")
            continue
        print(f"| {r['workload']} | {r['shape'][0]}x{r['shape'][1]} | " + " | ".join(
            f"{r[c]['GB/s']:.0f} ({r[c]['frac']:.2f})" for c in cols) + " |")
    with open(args.sweep, "w") as f:
        json.dump({"peak_gbs": peak, "peak_source": peak_src, "rows": rows}, f, indent=1)
    return 0


def run_linear(args):
    """W4A16 linear on the pages' weights (4096 x 4096, 14336 x 4096) under 1 .. 8192 tokens of
    N(0, 1) activations.  Roofline per shape: the larger of 2MNK / measured bf16 peak and
    (x + packed weight + y bytes) / measured HBM peak; frac = that time / measured time.
    Beside it: the pages' own order of work (nvfp4_dequantize into a bf16 buffer, then torch's
    bf16 linear) and a bf16 linear on an unquantized bf16 weight.  Before each rep L2 is
    flushed by a read of a 512 MB buffer (a read leaves no dirty lines whose write-back would
    land inside the timed window); CUDA events; median of 15 reps.  The timing floor of this
    method is reported beside the table: a one-element torch op (one empty launch) timed the
    same way."""
    import numpy as np
    import torch
    from qat_nvfp4_b200 import nvfp4 as nv
    from qat_nvfp4_b200 import synthetic

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm, hbm_src = hbm_peak()
    tc, tc_src = bf16_peak()
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def timed(fn, reps=15):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.sum(dtype=torch.int32)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        return sorted(ts)[len(ts) // 2] / 1e3

    one = torch.zeros(1, dtype=torch.float32, device=dev)
    floor_us = timed(lambda: one.add_(1.0), reps=31) * 1e6
    rows = []
    for (N, K) in [(4096, 4096), (14336, 4096)]:
        w = synthetic.activation_normal_device((N, K), 7, dev) * 0.02
        packed, scales, gs = nv.nvfp4_quantize(w, nv.nvfp4_amax(w))
        tiled = nv.nvfp4_w4a16_pack(packed, scales)
        wbuf = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        for M in (1, 4, 8, 16, 32, 128, 1024, 4096, 8192):
            x = synthetic.activation_normal_device((M, K), 8 + M, dev)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            lws = nv.nvfp4_w4a16_workspace(M, N, K, dev)
            where, tile_rows, splits = nv.nvfp4_w4a16_plan(M, N, K, lws.numel(), sms)
            kernel = f"{where} {tile_rows}" + (f" x{splits} K" if splits > 1 else "")
            t_fused = timed(lambda: nv.nvfp4_w4a16_linear(x, tiled, gs, N, out=y, workspace=lws))
            t_pages = timed(lambda: (nv.nvfp4_dequantize(packed, scales, gs, out=wbuf), torch.matmul(x, wbuf.t(), out=y)))
            t_bf16 = timed(lambda: torch.matmul(x, w.t(), out=y))
            flops = 2.0 * M * N * K
            nbytes = 2.0 * M * K + 0.5625 * N * K + 2.0 * M * N
            ideal = max(flops / (tc * 1e12), nbytes / (hbm * 1e9))
            cpu_us = None
            if M == 16:  # the oracle's forward (C dequantize + float64 matmul), one call on the host
                import oracle
                xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
                pk, sc, g = packed.cpu().numpy(), scales.cpu().numpy(), float(gs.item())
                t0 = time.perf_counter()
                oracle.w4a16_linear(xb, pk, sc, g, N)
                cpu_us = (time.perf_counter() - t0) * 1e6
            rows.append({"weight": [N, K], "tokens": M, "fused_us": t_fused * 1e6, "oracle_cpu_us": cpu_us,
                         "TFLOP/s": flops / t_fused / 1e12, "GB/s": nbytes / t_fused / 1e9,
                         "bound": "tensor" if flops / (tc * 1e12) >= nbytes / (hbm * 1e9) else "hbm",
                         "frac": ideal / t_fused, "dequant_then_linear_us": t_pages * 1e6,
                         "bf16_linear_us": t_bf16 * 1e6, "kernel": kernel})
            del x, y
        del w, packed, scales, tiled, wbuf
    print(f"bf16 peak {tc:.1f} TFLOP/s ({tc_src}); HBM peak {hbm:.1f} GB/s ({hbm_src}); "
          f"timing floor (one empty launch after the flush) {floor_us:.1f} us")
    print("| weight | tokens | W4A16 us | TFLOP/s | GB/s | bound | frac of roofline | dequantize + linear us "
          "| bf16 linear (unquantized weight) us | CPU oracle us (1 thread) | kernel (weight in, rows of x per tile, K split) |")
    print("|---|---|---|---|---|---|---|---|---|---|---|")
    for r in rows:
        cpu = f"{r['oracle_cpu_us']:.0f}" if r["oracle_cpu_us"] is not None else ""
        print(f"| {r['weight'][0]}x{r['weight'][1]} | {r['tokens']} | {r['fused_us']:.1f} | {r['TFLOP/s']:.0f} | "
              f"{r['GB/s']:.0f} | {r['bound']} | {r['frac']:.2f} | {r['dequant_then_linear_us']:.1f} | "
              f"{r['bf16_linear_us']:.1f} | {cpu} | {r['kernel']} |")
    with open(args.linear, "w") as f:
        json.dump({"bf16_tflops": tc, "hbm_gbs": hbm, "timing_floor_us": floor_us, "rows": rows}, f, indent=1)
    return 0


def run_strided(args):
    """amax, quantize and in-place fake-quant of row-strided views: the q, k and v columns
    (4096, 1024, 1024 wide) of a fused projection output of 16384 tokens (row stride 6144),
    each > L2, against the same calls on contiguous copies of the views.  GB/s counts the
    algorithmic bytes of the view (2, 2.5625 and 4 per element); CUDA events, median of 15,
    L2 flushed by a 512 MB read before each rep."""
    import torch
    from qat_nvfp4_b200 import nvfp4 as nv
    from qat_nvfp4_b200 import synthetic

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_src = hbm_peak()
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, reps=15):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.sum(dtype=torch.int32)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        return sorted(ts)[len(ts) // 2] / 1e3

    T, widths = 16384, (4096, 1024, 1024)
    fused = synthetic.activation_normal_device((T, sum(widths)), 21, dev)
    rows, c0 = [], 0
    for name, w in zip(("q", "k", "v"), widths):
        view = fused[:, c0:c0 + w]
        c0 += w
        copy = view.contiguous()
        n = view.numel()
        amax = nv.nvfp4_amax(view)
        packed = torch.empty((T, w // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((T, w // 16), dtype=torch.uint8, device=dev)
        gs = torch.empty(1, dtype=torch.float32, device=dev)
        r = {"view": name, "shape": [T, w], "row_stride": sum(widths)}
        for label, x in (("strided", view), ("contiguous", copy)):
            a = torch.empty(1, dtype=torch.float32, device=dev)
            keep = x.clone()
            t_amax = timed(lambda: nv.nvfp4_amax(x, out=a))
            t_q = timed(lambda: nv.nvfp4_quantize(x, amax, packed, scales, gs))
            t_fq = timed(lambda: nv.nvfp4_fake_quant(x, amax, out=x))  # in place, as a QAT forward on a view
            x.copy_(keep)
            for op, t, bpe in (("amax", t_amax, 2.0), ("quantize", t_q, 2.5625), ("fake_quant", t_fq, 4.0)):
                r[f"{op}_{label}_us"] = t * 1e6
                r[f"{op}_{label}_gbs"] = n * bpe / t / 1e9
        rows.append(r)
    print(f"HBM peak {peak:.1f} GB/s ({peak_src})")
    print("| view | shape (row stride) | op | strided us | GB/s (frac) | contiguous copy us | GB/s (frac) |")
    print("|---|---|---|---|---|---|---|")
    for r in rows:
        for op in ("amax", "quantize", "fake_quant"):
            gs_s, gs_c = r[f"{op}_strided_gbs"], r[f"{op}_contiguous_gbs"]
            print(f"| {r['view']} | {r['shape'][0]}x{r['shape'][1]} ({r['row_stride']}) | {op} | "
                  f"{r[f'{op}_strided_us']:.1f} | {gs_s:.0f} ({gs_s / peak:.2f}) | "
                  f"{r[f'{op}_contiguous_us']:.1f} | {gs_c:.0f} ({gs_c / peak:.2f}) |")
    with open(args.strided, "w") as f:
        json.dump({"hbm_gbs": peak, "rows": rows}, f, indent=1)
    return 0


def run_linear_shape(args):
    import torch
    from qat_nvfp4_b200 import nvfp4 as nv
    from qat_nvfp4_b200 import synthetic

    M, K, N = (int(v) for v in args.linear_shape.split(","))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    x = synthetic.activation_normal_device((M, K), 1, dev)
    w = synthetic.activation_normal_device((N, K), 2, dev) * 0.02
    packed, scales, gs = nv.nvfp4_quantize(w, nv.nvfp4_amax(w))
    tiled = nv.nvfp4_w4a16_pack(packed, scales)
    ws = nv.nvfp4_w4a16_workspace(M, N, K, dev)
    for _ in range(3):
        y = nv.nvfp4_w4a16_linear(x, tiled, gs, N, workspace=ws)
    torch.cuda.synchronize(dev)
    if nv.nvfp4_workspace_check(ws[:nv.WORKSPACE_BYTES]) != 0:
        raise SystemExit("W4A16 linear reported a timeout")
    print(json.dumps({"linear_shape": [M, K, N], "y_abs_mean": float(y.float().abs().mean())}))
    return 0


def main():
    args = parse_args()
    if args.sweep:
        return run_sweep(args)
    if args.linear:
        return run_linear(args)
    if args.linear_shape:
        return run_linear_shape(args)
    if args.strided:
        return run_strided(args)
    if args.cols < 1 or args.rows < 1:
        raise SystemExit("--rows and --cols must be positive")
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
