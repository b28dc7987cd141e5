"""Benchmark of the NVFP4 W4A4 hot path on B200.

One step = the whole path on one batch: tensor amax -> Four-Over-Six (MSE,
fp8_max 256) quantization of X -> NVFP4 GEMM against a pre-quantized weight
(scale-6, fp8_max 448) -> bf16 Y, on the long-prefill MLP shape
(X 32768 x 5120, W 17408 x 5120), as one nvfp4_quantize_gemm call (each
kernel a programmatic dependent of the one before it).  The breakdown times
the same step as two calls with an event between quantize and GEMM.  `value` is whole-job GEMM-equivalent
throughput, 2*M*N*K per step per GPU summed over ranks / step time (TFLOP/s);
the JSON line also carries the quantizer's GB/s and the GEMM's TFLOP/s with
their roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun) every rank runs an independent replica on its own X
(weak scaling: the path shards by tokens with W replicated and needs no
collective); times are the max over ranks.  `--impl reference` times the CPU
oracle (the plain, slow definition) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
METRIC = "quantize GB/s (% HBM peak); W4A4 GEMM TFLOPS (% dense NVFP4 peak)"
QUANT_BYTES_PER_ELEM = 2.5625   # read bf16 + write 0.5 B codes + 1/16 B scale
AMAX_BYTES_PER_ELEM = 2.0
# A ~0.2 ms spin on the GPU (torch.cuda._sleep) before each timed step, outside
# the events: the host's launch overhead then overlaps GPU work instead of
# showing up as idle time between the start event and the first kernel.
HOST_LEAD_CYCLES = 400_000
# dram__bytes_read.sum + dram__bytes_write.sum of one gemm_kernel launch on the
# full-size prefill workload (one-pass ncu capture), recorded with the SHA-1 of
# the kernel's sources at capture time; the bench reports it only while those
# sources are unchanged
GEMM_PREFILL_TRAFFIC = {"bytes": 1.4525e9, "read": 0.3500e9, "write": 1.1024e9,
                        "algorithmic": 1.285e9, "captured": "2026-12-03",
                        "kernel_sources_sha1": "1ad0301779ee3c0997b38e4fd2ef46c9058658ac",
                        "source": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,"
                                  "gpu__time_duration.sum (one pass) of gemm_kernel, prefill workload"}
GEMM_KERNEL_SOURCES = ("w4a4_gemm_nvfp4_b200/csrc/gemm.cu", "w4a4_gemm_nvfp4_b200/csrc/common.cuh",
                       "w4a4_gemm_nvfp4_b200/csrc/block_step.cuh")


def gemm_sources_sha1() -> str:
    h = hashlib.sha1()
    for rel in GEMM_KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(args):
    """The recorded per-launch DRAM traffic of the GEMM, or None when the
    workload is not the full-size prefill one or the kernel's sources changed
    since the capture."""
    if args.workload != "prefill" or args.x_rows:
        return None
    if GEMM_PREFILL_TRAFFIC["kernel_sources_sha1"] != gemm_sources_sha1():
        return None
    return GEMM_PREFILL_TRAFFIC


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p["bf16_tflops_sustained"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


class ClockSampler:
    """GPU clock / throttle samples taken while the timed region runs: an NVML
    thread polling every 5 ms (nvidia-smi as a fallback)."""

    REASONS = {  # NVML clocks-event reason bits
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self.error = None
        self.match = None

    def _handle(self, pynvml):
        """NVML handle of the CUDA device being timed.  NVML numbers every GPU
        of the machine, CUDA only the visible ones, so the two indexes can
        differ; the UUID names the same GPU in both."""
        try:
            u = str(torch.cuda.get_device_properties(self.gpu).uuid)
            self.match = "uuid"
            return pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:
            self.match = "index"
            return pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _run(self):
        import pynvml

        h = self._handle(pynvml)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self._stop.is_set():
            self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
            try:
                bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            except AttributeError:
                bits = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
            for name, bit in self.REASONS.items():
                if bits & bit:
                    self.reasons.add(name)
            self._stop.wait(0.005)

    def __enter__(self):
        import threading

        try:
            import pynvml

            pynvml.nvmlInit()
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # no NVML: report why
            self.error = f"nvml unavailable: {e}"
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": [self.error or "no samples"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(self.samples), "reasons": sorted(self.reasons),
                "samples": len(self.samples), "nvml_device_by": self.match}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def workload_of(args):
    """The named workload; --x-rows replaces the number of X rows (smaller
    captures of the same kernels)."""
    wl = workloads.WORKLOADS[args.workload]
    if args.x_rows:
        wl = dataclasses.replace(wl, x=dataclasses.replace(wl.x, rows=args.x_rows))
    return wl


def rank_x_operand(wl, rank: int):
    """Rank r's activations: the workload's X recipe with its own seed (weak
    scaling: every rank quantizes and multiplies a different X, same W)."""
    return workloads.Operand(**{**wl.x.__dict__, "seed": wl.x.seed + 101 * rank})


def spread(ts) -> dict:
    """Median, 10th and 90th percentile (nearest rank) of per-step times, ms."""
    xs = sorted(ts)
    pick = lambda q: xs[min(len(xs) - 1, max(0, int(round(q * (len(xs) - 1)))))]
    return {"median": round(statistics.median(xs), 4), "p10": round(pick(0.1), 4), "p90": round(pick(0.9), 4),
            "n": len(xs)}


def job_tflops(world: int, flops_per_rank: float, ms_max: float) -> float:
    """Whole-job throughput: all ranks' flops over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def _max_over_ranks(world, value: float, device) -> float:
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- ours --

def run_ours(args, world, rank, local):
    import w4a4_gemm_nvfp4_b200 as nv

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = workload_of(args)
    traffic = recorded_traffic(args)
    xm, xr, xF = args.x_recipe
    wm, wr, wF = wl.w_recipe
    M, N, K = wl.M, wl.N, wl.K
    # each rank gets its own activations (weak scaling), same weights
    xop = rank_x_operand(wl, rank)
    x_host = xop.make().pin_memory()
    x = x_host.to(device)
    w = wl.w.make().to(device)
    qw = nv.quantize(w, wm, wr, wF)               # offline weight quantization
    del w
    qx = nv.quantize(x, xm, xr, xF)
    q6 = nv.quantize(x, "six", "max", 448.0)      # scale-6 comparison buffers
    y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    gws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush_rd = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=device)
    flush_sum = torch.zeros((), dtype=torch.int64, device=device)

    def flush_l2(i):
        # write 256 MiB (evicts everything), then read another 256 MiB so the
        # write-backs of those dirty lines happen here, untimed, and the timed
        # kernels start from a cold but clean L2
        flush.fill_(i & 0xFF)
        torch.sum(flush_rd, dim=0, out=flush_sum)
    stream = torch.cuda.current_stream(device)

    def step(qbuf, mode, rule, F, ev=None):
        if ev:
            ev[0].record(stream)
        nv.quantize(x, mode, rule, F, out=qbuf)
        if ev:
            ev[1].record(stream)
        nv.gemm(qbuf, qw, out_dtype=torch.bfloat16, out=y, workspace=gws)
        if ev:
            ev[2].record(stream)

    def fused_step():
        # the whole path in one call: amax -> quantize X -> GEMM, each kernel
        # a programmatic dependent of the one before it
        nv.quantize_gemm(x, qw, xm, xr, xF, out_dtype=torch.bfloat16, x_out=qx, out=y, workspace=gws)

    for _ in range(args.warmup):
        fused_step()
        step(qx, xm, xr, xF)
        step(q6, "six", "max", 448.0)
    torch.cuda.synchronize()
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(gws) == nv.OK

    def timed_fused(steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush_l2(i)                             # L2 flush between steps (untimed)
            torch.cuda._sleep(HOST_LEAD_CYCLES)     # GPU busy while the host enqueues the step
            evs[i][0].record(stream)
            fused_step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    def timed(qbuf, mode, rule, F, steps):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(steps):
            flush_l2(i)                             # L2 flush between steps (untimed)
            torch.cuda._sleep(HOST_LEAD_CYCLES)     # GPU busy while the host enqueues the step
            step(qbuf, mode, rule, F, evs[i])
        torch.cuda.synchronize()
        tq = [e[0].elapsed_time(e[1]) for e in evs]
        tg = [e[1].elapsed_time(e[2]) for e in evs]
        return tq, tg

    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        steps_ms = timed_fused(args.steps)          # the headline: K whole steps
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(gws) == nv.OK
    # the breakdown, with its own clock samples (a long breakdown can run
    # warmer, and so slower, than the headline steps)
    bclocks = ClockSampler(local).__enter__()
    # the breakdown: the same step as two calls with an event between them
    _barrier(world)
    torch.cuda.synchronize()
    tq, tg = timed(qx, xm, xr, xF, args.steps)
    _barrier(world)
    torch.cuda.synchronize()
    tq6, tg6 = timed(q6, "six", "max", 448.0, args.steps)
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(gws) == nv.OK

    # the quantize kernel alone: alpha supplied (static), no amax pass
    qs = nv.quantize(x, xm, xr, global_scale=qx.global_scale)      # shares qx's alpha
    qs6 = nv.quantize(x, "six", "max", global_scale=q6.global_scale)

    def time_op(fn, steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for i in range(steps):
            flush_l2(i)
            torch.cuda._sleep(HOST_LEAD_CYCLES)
            evs[i][0].record(stream)
            fn()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    _barrier(world)
    torch.cuda.synchronize()
    t_qstatic = time_op(lambda: nv.quantize(x, xm, xr, out=qs, global_scale=qx.global_scale), args.steps)
    t_qstatic6 = time_op(lambda: nv.quantize(x, "six", "max", out=qs6, global_scale=q6.global_scale),
                         args.steps)
    assert nv.device_status(qs.workspace) == nv.OK and nv.device_status(qs6.workspace) == nv.OK
    ms_qstatic = _max_over_ranks(world, statistics.mean(t_qstatic), device)
    ms_qstatic6 = _max_over_ranks(world, statistics.mean(t_qstatic6), device)

    # the "next" entry points on the same operands: the GEMM writing Y as an
    # NVFP4 operand (4/6-MSE at a static output alpha), and the augmented-
    # channel step (ARCQuant: 128 residual channels of the most outlying
    # columns, then the GEMM over K + 128 against the weight with those
    # columns duplicated)
    S_ARC = 128
    y_alpha = (y.float().abs().amax() / (6 * 256.0)).reshape(1).to(torch.float32)
    qy = nv.gemm_quantized(qx, qw, y_alpha, "four_over_six", "mse")
    perm = x.float().abs().amax(dim=0).argsort(descending=True).to(torch.int32)
    qw_arc = nv.quantize_arc(wl.w.make().to(device), perm, S_ARC, nv.AUG_DUPLICATE, wm, wr, wF)
    qa = nv.quantize_arc(x, perm, S_ARC, nv.AUG_RESIDUAL, xm, xr, xF)
    y_arc = torch.empty_like(y)
    _barrier(world)
    torch.cuda.synchronize()
    ms_qout = time_op(lambda: nv.gemm_quantized(qx, qw, y_alpha, "four_over_six", "mse", out=qy), args.steps)
    ms_arc_q = time_op(lambda: nv.quantize_arc(x, perm, S_ARC, nv.AUG_RESIDUAL, xm, xr, xF, out=qa), args.steps)
    # the same with the activations' RMSNorm fused ahead (seeded gains near 1)
    gains = (1.0 + 0.25 * torch.randn(K, generator=torch.Generator().manual_seed(7))).to(torch.bfloat16).to(device)
    qn = nv.quantize_arc_rmsnorm(x, gains, 1e-6, perm, S_ARC, xm, xr, xF)
    ms_arc_norm = time_op(lambda: nv.quantize_arc_rmsnorm(x, gains, 1e-6, perm, S_ARC, xm, xr, xF, out=qn),
                          args.steps)

    def arc_step():  # the augmented layer in one call, as the headline step is
        nv.quantize_arc_gemm(x, perm, S_ARC, qw_arc, xm, xr, xF, out_dtype=torch.bfloat16, x_out=qa, out=y_arc,
                             workspace=gws)

    # the augmented step against the plain step, alternated in one loop so
    # that both see the same clocks
    t_plain_pair, t_arc_pair = [], []
    for i in range(args.steps):
        t_plain_pair += time_op(fused_step, 1)
        t_arc_pair += time_op(arc_step, 1)
    ms_arc_step = t_arc_pair
    assert (nv.device_status(qy.workspace) == nv.OK and nv.device_status(qa.workspace) == nv.OK
            and nv.device_status(qn.workspace) == nv.OK and nv.device_status(gws) == nv.OK)
    ms_plain_pair = _max_over_ranks(world, statistics.mean(t_plain_pair), device)
    ms_qout = _max_over_ranks(world, statistics.mean(ms_qout), device)
    ms_arc_q = _max_over_ranks(world, statistics.mean(ms_arc_q), device)
    ms_arc_norm = _max_over_ranks(world, statistics.mean(ms_arc_norm), device)
    ms_arc_step = _max_over_ranks(world, statistics.mean(ms_arc_step), device)
    del qy, qa, qn, qw_arc, y_arc
    bclocks.__exit__(None, None, None)

    ms_step = _max_over_ranks(world, statistics.mean(steps_ms), device)
    ms_two_calls = _max_over_ranks(world, statistics.mean(a + b for a, b in zip(tq, tg)), device)
    ms_quant = _max_over_ranks(world, statistics.mean(tq), device)
    ms_gemm = _max_over_ranks(world, statistics.mean(tg), device)
    ms_quant6 = _max_over_ranks(world, statistics.mean(tq6), device)

    # end to end through the public API with host buffers: every step copies
    # its X in from pinned host memory and its Y back out.  Two steps are in
    # flight, each with its own device X and Y: the copies in, the one-call
    # layer and the copies out run on three streams, so one step's copies
    # overlap the other's compute and the two copy directions overlap each
    # other (PCIe is full duplex).
    slots = 2
    x_dev = [x] + [torch.empty_like(x) for _ in range(slots - 1)]
    y_dev = [y] + [torch.empty_like(y) for _ in range(slots - 1)]
    y_host = [torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True) for _ in range(slots)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(slots)]
    ev_done = [torch.cuda.Event() for _ in range(slots)]
    ev_out = [torch.cuda.Event() for _ in range(slots)]
    e2e_steps = max(1, min(args.steps, 8))
    _barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(e2e_steps):
        k = i % slots
        with torch.cuda.stream(s_in):
            if i >= slots:
                s_in.wait_event(ev_done[k])          # the slot's last compute has read its X
            x_dev[k].copy_(x_host, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if i >= slots:
            stream.wait_event(ev_out[k])             # the slot's last Y has been copied out
        nv.quantize_gemm(x_dev[k], qw, xm, xr, xF, out_dtype=torch.bfloat16, x_out=qx, out=y_dev[k],
                         workspace=gws)
        ev_done[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[k])
            y_host[k].copy_(y_dev[k], non_blocking=True)
            ev_out[k].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(gws) == nv.OK
    ms_e2e = _max_over_ranks(world, e0.elapsed_time(e1) / e2e_steps, device)
    del x_dev, y_dev, y_host

    flops = 2.0 * M * N * K
    peaks = _peaks()
    fp4_peak = 4.0 * peaks["bf16"]
    gemm_tflops = flops / (ms_gemm * 1e-3) / 1e12
    quant_gbs = (QUANT_BYTES_PER_ELEM + AMAX_BYTES_PER_ELEM) * M * K / (ms_quant * 1e-3) / 1e9
    value = job_tflops(world, flops, ms_step)
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4",
        "data": "synthetic (seeded; shapes of the pages' long-prefill MLP workload)",
        "config": {
            "workload": f"{args.workload}: X {M}x{K} bf16 (4/6-{xr}, fp8_max {xF:g}) -> GEMM with "
                        f"W {N}x{K} pre-quantized ({wm}, fp8_max {wF:g}) -> Y bf16",
            "M": M, "N": N, "K": K, "per_gpu_batch_tokens": M,
            "parallelism": f"replicas x{world}",
            "l2": "flushed between steps (256 MiB write, then 256 MiB read so the timed kernels do not pay the write-backs; untimed)",
        },
        "roofline": {
            "bound": "tensor",
            "kernel": "gemm_kernel",
            "achieved": round(gemm_tflops, 1),
            "peak": round(fp4_peak, 1),
            "unit": "TFLOP/s",
            "frac": round(gemm_tflops / fp4_peak, 4),
            "peak_source": f"4 x {peaks['source']} bf16 burst ({peaks['bf16']} TF/s)",
            # recorded from an ncu capture of this kernel version, not measured here
            "traffic": traffic["bytes"] if traffic else None,
            "traffic_detail": traffic if traffic else {
                "why_null": "no capture of the current kernel sources on this workload",
                "kernel_sources_sha1": gemm_sources_sha1()},
        },
        "breakdown": {
            "ms_step_two_calls": round(ms_two_calls, 4),
            "ms_quantize_46": round(ms_quant, 4),
            "ms_quantize_six": round(ms_quant6, 4),
            "overhead_46_vs_six": round(ms_quant / ms_quant6 - 1.0, 4),
            "quantize_end_to_end_GBps": round(quant_gbs, 1),
            "quantize_frac_hbm": round(quant_gbs / peaks["hbm"], 4),
            "ms_quantize_kernel_46_static_alpha": round(ms_qstatic, 4),
            "ms_quantize_kernel_six_static_alpha": round(ms_qstatic6, 4),
            "quantize_kernel_46_GBps": round(QUANT_BYTES_PER_ELEM * M * K / (ms_qstatic * 1e-3) / 1e9, 1),
            "quantize_kernel_46_frac_hbm": round(
                QUANT_BYTES_PER_ELEM * M * K / (ms_qstatic * 1e-3) / 1e9 / peaks["hbm"], 4),
            "overhead_46_vs_six_kernel": round(ms_qstatic / ms_qstatic6 - 1.0, 4),
            "hbm_peak_GBps": peaks["hbm"],
            "ms_gemm": round(ms_gemm, 4),
            "gemm_TFLOPs": round(gemm_tflops, 1),
            "ms_gemm_after_six": round(_max_over_ranks(world, statistics.mean(tg6), device), 4),
            "ms_gemm_nvfp4_out_46mse": round(ms_qout, 4),
            "gemm_nvfp4_out_TFLOPs": round(flops / (ms_qout * 1e-3) / 1e12, 1),
            "gemm_nvfp4_out_frac_fp4_peak": round(flops / (ms_qout * 1e-3) / 1e12 / fp4_peak, 4),
            "ms_quantize_arc_S128": round(ms_arc_q, 4),
            "ms_quantize_arc_rmsnorm_S128": round(ms_arc_norm, 4),
            "ms_step_arc_S128": round(ms_arc_step, 4),
            "ms_step_beside_arc": round(ms_plain_pair, 4),
            "arc_step_overhead_vs_step": round(ms_arc_step / ms_plain_pair - 1.0, 4),
        },
        "clocks_breakdown": bclocks.summary(),
        "stats": {
            "what": "per-step CUDA-event times of this rank (rank 0), ms",
            "ms_per_step": spread(steps_ms),
            "ms_quantize_46": spread(tq),
            "ms_gemm": spread(tg),
            "ms_quantize_kernel_46_static_alpha": spread(t_qstatic),
            "ms_quantize_kernel_six_static_alpha": spread(t_qstatic6),
        },
        "e2e": {
            "value": round(job_tflops(world, flops, ms_e2e), 2),
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": M * K * 2,
            "d2h_bytes_per_step": M * N * 2,
            "ms_per_step": round(ms_e2e, 3),
            "how": f"{e2e_steps} steps, two in flight: X in on one copy stream, the one-call layer, Y out on "
                   "another (pinned host buffers)",
        },
        "gpu_launches": 3 * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args, sample_rows=1024)  # about 40 s of CPU work in all
    return result


# ------------------------------------------------------------ oracle (CPU) --

def _oracle_sample(wl, xr_recipe, rows, w_deq=None):
    """One bounded oracle pass: quantize `rows` rows of X (4/6 rule) and
    their fp64 GEMM against the oracle-quantized W.  Returns flops done."""
    import numpy as np

    import oracle

    mode = {"six": oracle.MODE_SIX, "four_over_six": oracle.MODE_FOUR_OVER_SIX}
    rule = {"max": oracle.RULE_MAX, "mae": oracle.RULE_MAE, "mse": oracle.RULE_MSE}
    xm, xr, xF = xr_recipe
    x = workloads.Operand(**{**wl.x.__dict__, "rows": rows}).make()
    xc, xs, xa = oracle.quantize(x, mode[xm], rule[xr], xF)
    xd = oracle.dequantize(xc, xs, xa)
    _ = xd @ w_deq.T
    return 2.0 * rows * w_deq.shape[0] * wl.K


def _w_dequant(wl):
    import oracle

    mode = {"six": oracle.MODE_SIX, "four_over_six": oracle.MODE_FOUR_OVER_SIX}
    rule = {"max": oracle.RULE_MAX, "mae": oracle.RULE_MAE, "mse": oracle.RULE_MSE}
    wm, wr, wF = wl.w_recipe
    wc, ws, wa = oracle.quantize(wl.w.make(), mode[wm], rule[wr], wF)
    return oracle.dequantize(wc, ws, wa)


def _cores():
    """Threads the oracle sample runs on: the fp64 GEMM's BLAS pool (the C
    quantizer is single-threaded and the smaller part), else the CPU affinity."""
    try:
        import numpy  # noqa: F401  (loads the BLAS library threadpoolctl inspects)
        from threadpoolctl import threadpool_info

        blas = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if blas:
            return max(blas)
    except Exception:
        pass
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def _host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_quantizer_baseline(wl, x_recipe):
    """The oracle quantizer on the workload's whole X: amax, then every block,
    single-threaded and on all host threads (row slices, one oracle call per
    slice; ctypes releases the GIL during each), results checked identical.
    GB/s over the same 4.5625 B/element as the GPU's end-to-end figure."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle

    mode = {"six": oracle.MODE_SIX, "four_over_six": oracle.MODE_FOUR_OVER_SIX}
    rule = {"max": oracle.RULE_MAX, "mae": oracle.RULE_MAE, "mse": oracle.RULE_MSE}
    xm, xr, xF = x_recipe
    x = wl.x.make()
    rows, K = x.shape
    bits = oracle.as_bf16_bits(x)
    t0 = time.perf_counter()
    amax, _ = oracle.amax(bits)
    alpha = oracle.global_scale(amax, xF)
    t_amax = time.perf_counter() - t0
    t0 = time.perf_counter()
    c1, s1 = oracle.quantize_rows(bits, alpha, mode[xm], rule[xr])
    t1 = time.perf_counter() - t0 + t_amax
    threads = _host_threads()
    edges = np.linspace(0, rows, threads + 1).astype(int)
    t0 = time.perf_counter()
    amax_n, _ = oracle.amax(bits)   # the amax pass again, inside the multi-threaded time
    with ThreadPoolExecutor(threads) as pool:
        parts = list(pool.map(lambda i: oracle.quantize_rows(bits[edges[i]:edges[i + 1]], alpha, mode[xm], rule[xr]),
                              range(threads)))
    tn = time.perf_counter() - t0
    identical = (amax_n == amax and np.array_equal(np.concatenate([p[0] for p in parts]), c1)
                 and np.array_equal(np.concatenate([p[1] for p in parts]), s1))
    nbytes = (QUANT_BYTES_PER_ELEM + AMAX_BYTES_PER_ELEM) * rows * K
    return {"GBps_1_thread": round(nbytes / t1 / 1e9, 4), "GBps_all_threads": round(nbytes / tn / 1e9, 4),
            "threads": threads, "s_1_thread": round(t1, 2), "s_all_threads": round(tn, 2),
            "identical": bool(identical),
            "sample": f"the whole X ({rows}x{K}, {xm}-{xr}, fp8_max {xF:g}): amax + every block; the "
                      f"multi-threaded run splits the rows over {threads} threads"}


def cpu_gemm_baseline(wl, x_recipe, rows=256):
    """The oracle GEMM (fp64 matmul of the exactly dequantized operands) on a
    slice of `rows` rows of X; the full-size time is extrapolated."""
    import oracle

    mode = {"six": oracle.MODE_SIX, "four_over_six": oracle.MODE_FOUR_OVER_SIX}
    rule = {"max": oracle.RULE_MAX, "mae": oracle.RULE_MAE, "mse": oracle.RULE_MSE}
    xm, xr, xF = x_recipe
    w_deq = _w_dequant(wl)
    x = workloads.Operand(**{**wl.x.__dict__, "rows": rows}).make()
    xc, xs, xa = oracle.quantize(x, mode[xm], rule[xr], xF)
    t0 = time.perf_counter()
    xd = oracle.dequantize(xc, xs, xa)
    _ = xd @ w_deq.T
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * wl.N * wl.K
    return {"GFLOPs": round(flops / dt / 1e9, 2), "rows": rows, "threads": _cores(), "s": round(dt, 3),
            "full_size_s_extrapolated": round(dt * wl.M / rows, 1),
            "sample": f"{rows} rows of X dequantized and multiplied in fp64 by the dequantized W {wl.N}x{wl.K} "
                      f"(BLAS threads {_cores()}); the full-size time is that x {wl.M}/{rows}, extrapolated"}


def cpu_baseline(args, sample_rows=64):
    """The oracle timed on this host: a bounded sample of the whole step
    (quantize `sample_rows` rows of X, then their fp64 GEMM against the
    dequantized W) as the headline figure, plus the quantizer on the whole X
    and the GEMM on a 256-row slice as separate records."""
    wl = workload_of(args)
    w_deq = _w_dequant(wl)
    t0 = time.perf_counter()
    flops = _oracle_sample(wl, args.x_recipe, sample_rows, w_deq)
    dt = time.perf_counter() - t0
    del w_deq
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(),
            "kind": "oracle",
            "sample": f"{sample_rows} rows of X ({wl.K} wide) quantized by the C oracle (1 thread) + "
                      f"fp64 numpy GEMM against the oracle-dequantized W {wl.N}x{wl.K} "
                      f"({_cores()} BLAS threads); W quantization untimed; {dt:.1f} s",
            "quantizer": cpu_quantizer_baseline(wl, args.x_recipe),
            "gemm": cpu_gemm_baseline(wl, args.x_recipe)}


def run_reference(args, world, rank):
    wl = workload_of(args)
    w_deq = _w_dequant(wl)
    rows = args.cpu_rows
    for _ in range(args.warmup):
        _oracle_sample(wl, args.x_recipe, max(1, rows // 8), w_deq)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += _oracle_sample(wl, args.x_recipe, rows, w_deq)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = (f"each step: {rows} rows of X quantized by the C oracle (1 thread) + fp64 numpy "
              f"GEMM against the oracle-dequantized W {wl.N}x{wl.K} ({_cores()} BLAS threads)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantize + f64 GEMM",
        "data": "synthetic (seeded)",
        "config": {"workload": f"{args.workload} (oracle sample of {rows} X rows per step)",
                   "M": wl.M, "N": wl.N, "K": wl.K},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_sweep(args):
    """The quantizer sweep over the C2 shapes and recipes, and the GEMM of each
    configured workload: one JSON line per item (1 GPU; not the headline)."""
    import w4a4_gemm_nvfp4_b200 as nv

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    peaks = _peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush_rd = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=device)
    flush_sum = torch.zeros((), dtype=torch.int64, device=device)
    stream = torch.cuda.current_stream(device)

    def timed(fn, n):
        for _ in range(3):
            fn()
        ts = []
        for i in range(n):
            flush.fill_(i & 0xFF)
            torch.sum(flush_rd, dim=0, out=flush_sum)
            torch.cuda._sleep(HOST_LEAD_CYCLES)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    for rows, K in workloads.SWEEP_SHAPES:
        x = workloads.sweep_operand(rows, K, seed=0).make().to(device)
        six_kernel = None
        for m, r, F in workloads.SWEEP_RECIPES:
            q = nv.quantize(x, m, r, F)
            qs = nv.quantize(x, m, r, global_scale=q.global_scale)
            t_e2e = timed(lambda: nv.quantize(x, m, r, F, out=q), args.steps)
            t_k = timed(lambda: nv.quantize(x, m, r, out=qs, global_scale=q.global_scale), args.steps)
            assert nv.device_status(q.workspace) == nv.OK and nv.device_status(qs.workspace) == nv.OK
            if m == "six":
                six_kernel = t_k
            n = rows * K
            print(json.dumps({
                "sweep": "quantize", "rows": rows, "K": K, "recipe": f"{m}-{r}-{F:g}",
                "ms_kernel": round(t_k, 4), "GBps_kernel": round(QUANT_BYTES_PER_ELEM * n / t_k / 1e6, 1),
                "frac_hbm_kernel": round(QUANT_BYTES_PER_ELEM * n / t_k / 1e6 / peaks["hbm"], 4),
                "ms_end_to_end": round(t_e2e, 4),
                "GBps_end_to_end": round((QUANT_BYTES_PER_ELEM + AMAX_BYTES_PER_ELEM) * n / t_e2e / 1e6, 1),
                "overhead_vs_six_kernel": None if m == "six" else round(t_k / six_kernel - 1.0, 4),
                "l2": "flushed between iterations", "median_of": args.steps}), flush=True)
            # the other quantizer entry points, amax pass included: blocks down
            # the columns (x^T), and 128 augmented residual channels
            n_bytes = (QUANT_BYTES_PER_ELEM + AMAX_BYTES_PER_ELEM) * n
            qt = nv.quantize_t(x, m, r, F)
            t_t = timed(lambda: nv.quantize_t(x, m, r, F, out=qt), args.steps)
            assert nv.device_status(qt.workspace) == nv.OK
            S = 128
            perm = torch.randperm(K, generator=torch.Generator().manual_seed(5)).to(torch.int32).to(device)
            qa = nv.quantize_arc(x, perm, S, nv.AUG_RESIDUAL, m, r, F)
            t_a = timed(lambda: nv.quantize_arc(x, perm, S, nv.AUG_RESIDUAL, m, r, F, out=qa), args.steps)
            assert nv.device_status(qa.workspace) == nv.OK
            arc_bytes = (2.0 + AMAX_BYTES_PER_ELEM + (QUANT_BYTES_PER_ELEM - 2.0) * (K + S) / K) * n
            print(json.dumps({
                "sweep": "quantize_variants", "rows": rows, "K": K, "recipe": f"{m}-{r}-{F:g}",
                "ms_transposed": round(t_t, 4), "GBps_transposed": round(n_bytes / t_t / 1e6, 1),
                "ms_arc_S128": round(t_a, 4), "GBps_arc_S128": round(arc_bytes / t_a / 1e6, 1),
                "arc_overhead_vs_rows": round(t_a / t_e2e - 1.0, 4),
                "l2": "flushed between iterations", "median_of": args.steps}), flush=True)
            del qt, qa
        del x
        torch.cuda.empty_cache()
    fp4_peak = 4.0 * peaks["bf16"]
    for name in ("mlp8b", "attn27b", "prefill"):
        wl = workloads.WORKLOADS[name]
        xm, xr, xF = wl.x_recipes[-1]
        wm, wr, wF = wl.w_recipe
        x = wl.x.make().to(device)
        w = wl.w.make().to(device)
        qx = nv.quantize(x, xm, xr, xF)
        qw = nv.quantize(w, wm, wr, wF)
        y = torch.empty(wl.M, wl.N, dtype=torch.bfloat16, device=device)
        ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=device)
        t = timed(lambda: nv.gemm(qx, qw, out=y, workspace=ws), args.steps)
        assert nv.device_status(ws) == nv.OK
        tf = 2.0 * wl.M * wl.N * wl.K / t / 1e9
        print(json.dumps({
            "sweep": "gemm", "workload": name, "M": wl.M, "N": wl.N, "K": wl.K,
            "x_recipe": f"{xm}-{xr}-{xF:g}", "w_recipe": f"{wm}-{wr}-{wF:g}",
            "ms": round(t, 4), "TFLOPs": round(tf, 1), "frac_fp4_peak": round(tf / fp4_peak, 4),
            "l2": "flushed between iterations", "median_of": args.steps}), flush=True)
        # the GEMM variants on the same operands: two output-column segments
        # with their own B scales, and Y written as an NVFP4 operand (4/6-MSE)
        half = wl.N // 2 // 64 * 64
        b_globals = torch.stack([qw.global_scale[0]] * 2)
        t_seg = timed(lambda: nv.gemm_segmented(qx, qw, b_globals, [half, wl.N], out=y, workspace=ws),
                      args.steps)
        assert nv.device_status(ws) == nv.OK
        y_alpha = torch.tensor([max(float(y.abs().max()), 1e-30) / (6 * 256.0)], dtype=torch.float32,
                               device=device)
        qy = nv.gemm_quantized(qx, qw, y_alpha, "four_over_six", "mse")
        t_q = timed(lambda: nv.gemm_quantized(qx, qw, y_alpha, "four_over_six", "mse", out=qy), args.steps)
        assert nv.device_status(qy.workspace) == nv.OK
        flops = 2.0 * wl.M * wl.N * wl.K
        print(json.dumps({
            "sweep": "gemm_variants", "workload": name, "M": wl.M, "N": wl.N, "K": wl.K,
            "ms_segmented_2": round(t_seg, 4), "TFLOPs_segmented_2": round(flops / t_seg / 1e9, 1),
            "ms_nvfp4_out_46mse": round(t_q, 4), "TFLOPs_nvfp4_out_46mse": round(flops / t_q / 1e9, 1),
            "frac_fp4_peak_nvfp4_out": round(flops / t_q / 1e9 / fp4_peak, 4),
            "l2": "flushed between iterations", "median_of": args.steps}), flush=True)
        del x, w, qx, qw, y, qy
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill", choices=["prefill", "mlp8b", "attn27b", "pr1"])
    ap.add_argument("--x-recipe", default="four_over_six,mse,256",
                    help="mode,rule,fp8_max for X (default four_over_six,mse,256)")
    ap.add_argument("--cpu-rows", type=int, default=256, help="X rows per oracle step (reference arm)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--x-rows", type=int, default=0,
                    help="replace the workload's X rows (profiling captures of a smaller case)")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the headline step: the quantizer sweep and every GEMM workload, "
                         "one JSON line each (1 GPU)")
    args = ap.parse_args()
    m, r, f = args.x_recipe.split(",")
    args.x_recipe = (m, r, float(f))
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")

    world, rank, local = _dist()
    if args.sweep:
        if world == 1 and args.impl == "ours":
            run_sweep(args)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        res = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
