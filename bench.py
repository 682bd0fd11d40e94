"""Benchmark of the NVFP4 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload per_token|swiglu|swiglu_fp8|decode|decode_f32|prefill|tiny]
                    [--m 32] [--a-layout 128x4|8x4] [--configs auto|none|w1,w2]
                    [--no-cpu-baseline] [--no-all-cores] [--cpu-seconds 10]

Default workload: per-token NVFP4 quantize of X bf16 [8192, 7168] (N(0,1) with 0.1% of
entries x50), one fp32 global scale per token, E4M3 scales in the 128x4 layout. A step is
one call of the path on one batch; inputs are resident in HBM and rotated over enough
copies that no step finds its input in the 126 MB L2. The default run then measures the
GEMM half of the metric the same way -- the prefill GEMM 8192 x 8192 x 8192 and the decode
GEMM M = 32, N = 28672, K = 8192 (128x4 activation scales) -- and reports each, with its own
roofline, clocks, e2e and cpu_baseline, in the line's `configs` list.

Prints one JSON line (rank 0). `value` is whole-job throughput in the workload's unit
(GB/s of algorithmic bytes for the quantize kernels and the decode GEMMs, TFLOP/s for the
prefill and tiny GEMMs), measured with
CUDA events on the launching stream, max over ranks. Multi-GPU runs are independent
replicas (weak scaling): the path has no exchange step. `cpu_baseline` times the oracle on
a bounded sample on one host core, repeated for about --cpu-seconds, and, under
`all_cores`, on every host core.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 GEMM TFLOPS + quantize GB/s, each as % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0  # nominal dense ratio (9 PF fp4 / 2.25 PF bf16)
# Second denominators, reported beside the measured ones: the ~8 TB/s HBM3e figure the
# quantize targets are stated against, and the FP4 tensor-op counter peak of the chip
# (32768 flop per cycle per SM x 148 SMs x 1965 MHz).
NOMINAL_HBM_GBS = 8000.0
FP4_COUNTER_PEAK_TFLOPS = 32768 * 148 * 1965e6 / 1e12
# The sub-configurations a default run adds after its headline line (the GEMM half of the
# metric): the compute-bound prefill GEMM and the weight-streaming decode GEMM.
DEFAULT_CONFIGS = ("prefill", "decode")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------------------- workloads

def algorithmic(workload, M=None, K=None, N=None, H=None, a_layout="128x4"):
    """Algorithmic bytes (and FLOPs) of one launch: every input byte read once, every output
    byte written once."""
    if workload == "per_token":
        x = M * K * 2
        q = M * K // 2
        sf = (-(-M // 128) * 128) * (-(-(K // 16) // 4) * 4)
        g = M * 4
        return {"bytes": x + q + sf + g, "read": x, "written": q + sf + g, "flops": 0}
    if workload == "swiglu_fp8":
        x = M * 2 * H * 2
        q = M * H
        return {"bytes": x + q, "read": x, "written": q, "flops": 0}
    if workload == "swiglu":
        x = M * 2 * H * 2
        q = M * H // 2
        sf = (-(-M // 128) * 128) * (-(-(H // 16) // 4) * 4)
        return {"bytes": x + q + sf, "read": x, "written": q + sf, "flops": 0}
    if workload in ("decode", "prefill", "tiny", "decode_f32"):
        rows_a = (-(-M // 8) * 8) if a_layout == "8x4" else (-(-M // 128) * 128)
        a = M * K // 2 + rows_a * K // 16
        if workload == "decode_f32":  # fp32 activation scales [M, K/16]
            a = M * K // 2 + M * (K // 16) * 4
        w = N * K // 2 + (-(-N // 128) * 128) * K // 16
        out = M * N * 2
        return {"bytes": a + w + out, "read": a + w, "written": out, "flops": 2 * M * N * K}
    raise ValueError(workload)


class Clocks:
    """Samples the SM clock and the clock-event (throttle) reasons while the timed region runs.

    A thread polls NVML back to back (a query takes well under a millisecond), so even a
    timed region of a few milliseconds gets samples. One sample is also taken right before
    and right after the region; if the region was too short for the thread to land a sample
    inside it, those two bracketing samples are reported and `window` says so. Falls back
    to `nvidia-smi -lms 100` when NVML cannot be loaded."""

    REASONS = {  # NVML clocks-event reason bits
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, bus_id=None):
        self.bus_id = bus_id
        self.inside, self.bracket = [], []
        self.max_mhz = None
        self.nv = None
        self.handle = None
        self.thread = None
        self.stop = False

    def _sample(self):
        nv = self.nv
        try:
            mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
            fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            return (float(mhz), int(fn(self.handle)))
        except Exception:
            return None

    def _poll(self):
        while not self.stop:
            s = self._sample()
            if s is not None:
                self.inside.append(s)
            time.sleep(0.0002)

    def __enter__(self):
        if self.bus_id is None:
            return self
        try:
            import pynvml as nv

            nv.nvmlInit()
            self.nv = nv
            self.handle = nv.nvmlDeviceGetHandleByPciBusId(self.bus_id)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM))
        except Exception:
            self.nv = None
            return self
        s = self._sample()
        if s is not None:
            self.bracket.append(s)
        import threading

        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop = True
            self.thread.join()
            s = self._sample()
            if s is not None:
                self.bracket.append(s)
        if self.nv is not None:
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        rows, window = self.inside, "inside"
        if not rows:
            rows, window = self.bracket, "bracketing"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        reasons = sorted({name for _, bits in rows for name, b in self.REASONS.items() if bits & b})
        return {"sm_mhz": statistics.median(m for m, _ in rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows), "window": window, "source": "nvml"}


def _source_hash(*rel):
    h = hashlib.sha256()
    for r in rel:
        with open(os.path.join(ROOT, r), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source still matches."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e:
        return None
    if e.get("source_sha") != _source_hash(*e["sources"]):
        return None
    return e["bytes_per_launch"]


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(ms, dist, device):
    """The largest of every rank's time (the job is as slow as its slowest rank); `ms` as is
    with one rank. Every rank must call it, in the same order."""
    if dist is None:
        return ms
    import torch

    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_throughput(world, units_per_rank_step, ms_per_step):
    """Whole-job throughput: all ranks' units of one step over the slowest rank's step time."""
    return world * units_per_rank_step / (ms_per_step / 1e3)


# ----------------------------------------------------------------------------- our arm

def workload_config(wl, args):
    """The workload keys of the JSON line's config (shared by both arms)."""
    if wl == "per_token":
        return {"workload": "per-token NVFP4 quantize", "shape": [8192, 7168], "input": "bf16",
                "dist": "N(0,1), 0.1% of entries x50", "scales": "E4M3 128x4",
                "global_scale": "fp32 per token", "l2": "input rotated over 3 copies (352 MB > 126 MB L2)"}
    if wl == "swiglu":
        return {"workload": "fused SwiGLU + NVFP4 quantize", "shape": [4096, 2 * 14336],
                "input": "bf16", "dist": "N(0,1)", "scales": "E4M3 128x4",
                "global_scale": "fp32 per tensor", "l2": "input rotated over 2 copies (470 MB > 126 MB L2)"}
    if wl == "swiglu_fp8":
        return {"workload": "fused SwiGLU + FP8 E4M3 quantize", "shape": [4096, 2 * 14336],
                "input": "bf16", "dist": "N(0,1)", "output": "E4M3 [M, H], scale 448/60",
                "l2": "input rotated over 2 copies (470 MB > 126 MB L2)"}
    if wl in ("decode", "decode_f32"):
        M, N, K, ncopy = args.m, 28672, 8192, 2
    elif wl == "prefill":
        M, N, K, ncopy = 8192, 8192, 8192, 3
    elif wl == "tiny":
        M, N, K, ncopy = 16, 256, 512, 1
    else:
        raise SystemExit(f"unknown workload {wl}")
    return {"workload": f"NVFP4 GEMM ({wl})", "M": M, "N": N, "K": K,
            "a_scales": "fp32 [M, K/16]" if wl == "decode_f32" else args.a_layout,
            "w_scales": "128x4", "out": "fp16", "l2": f"operands rotated over {ncopy} copies"}


def run_ours(args, rank, world, torch, dist):
    import nvfp4_block_scaled_10_b200 as nv
    from nvfp4_block_scaled_10_b200 import build, workloads

    build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    wl = args.workload
    layout_code = nv.SF_8x4 if args.a_layout == "8x4" else nv.SF_128x4

    kernels_per_step = None  # all of this library's kernels a step launches, where more than one
    launch_scope = None      # what the roofline's per-launch time covers, where not the kernel alone

    # ---- inputs (resident in HBM, rotated so no step reuses L2-resident data)
    if wl == "per_token":
        M, K = 8192, 7168
        x_host = workloads.per_token(M, K, seed=workloads.SEEDS["per_token"] + rank)
        copies = [x_host.to(dev) for _ in range(3)]
        g = torch.empty(M, dtype=torch.float32, device=dev)
        q = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        sf = torch.empty(nv.nvfp4_sf_bytes(M, K, nv.SF_128x4), dtype=torch.uint8, device=dev)
        alg = algorithmic(wl, M=M, K=K)
        kernel_key, kernel_name = "quant_pertoken_regs", "quant_pertoken_regs_kernel"

        def step(i):
            nv.nvfp4_quantize(copies[i % 3], g, per_token=True, sf_layout=nv.SF_128x4, q=q, sf=sf)
        launches_per_step, period = 1, 3
        workload_desc = workload_config(wl, args)
        unit, factor = "GB/s", alg["bytes"] / 1e9
    elif wl == "swiglu":
        M, H = 4096, 14336
        x_host = workloads.swiglu(M, H, seed=workloads.SEEDS["swiglu"] + rank)
        copies = [x_host.to(dev) for _ in range(2)]
        gval = 2688.0 / 60.0  # encode scale of |Y| up to ~60; value only, not a timing input
        gdev = torch.tensor([gval], dtype=torch.float32, device=dev)
        q = torch.empty(M, H // 2, dtype=torch.uint8, device=dev)
        sf = torch.empty(nv.nvfp4_sf_bytes(M, H, nv.SF_128x4), dtype=torch.uint8, device=dev)
        alg = algorithmic(wl, M=M, H=H)
        kernel_key, kernel_name = "swiglu_quant", "swiglu_quant_kernel"

        def step(i):
            nv.swiglu_nvfp4_quantize(copies[i % 2], gdev, sf_layout=nv.SF_128x4, q=q, sf=sf)
        launches_per_step, period = 1, 2
        workload_desc = workload_config(wl, args)
        unit, factor = "GB/s", alg["bytes"] / 1e9
    elif wl == "swiglu_fp8":
        M, H = 4096, 14336
        x_host = workloads.swiglu(M, H, seed=workloads.SEEDS["swiglu"] + rank)
        copies = [x_host.to(dev) for _ in range(2)]
        sdev = torch.tensor([448.0 / 60.0], dtype=torch.float32, device=dev)
        q = torch.empty(M, H, dtype=torch.uint8, device=dev)
        sf = torch.empty(1, dtype=torch.uint8, device=dev)
        alg = algorithmic(wl, M=M, H=H)
        kernel_key, kernel_name = "swiglu_fp8", "swiglu_fp8_kernel"

        def step(i):
            nv.swiglu_fp8_quantize(copies[i % 2], sdev, q=q)
        launches_per_step, period = 1, 2
        workload_desc = workload_config(wl, args)
        unit, factor = "GB/s", alg["bytes"] / 1e9
    elif wl in ("decode", "prefill", "tiny", "decode_f32"):
        if wl in ("decode", "decode_f32"):
            M, N, K = args.m, 28672, 8192
            a_b, w_b = workloads.decode(M, N, K)
            ncopy = 2
        elif wl == "prefill":
            M = N = K = 8192
            a_b, w_b = workloads.prefill()
            ncopy = 3
        else:
            a_b, w_b = workloads.tiny()
            M, K = a_b.shape
            N = w_b.shape[0]
            ncopy = 1
        a_d, w_d = a_b.to(dev), w_b.to(dev)
        ga = nv.nvfp4_global_scale(a_d)
        gw = nv.nvfp4_global_scale(w_d)
        ops = []
        for _ in range(ncopy):
            if wl == "decode_f32":
                # the plugin contract: combined fp32 activation scales E4M3 x fp32(1 / ga) and a
                # multiplying weight scale fp32(1 / gw) (input preparation, not timed)
                aq, asf_lin, _ = nv.nvfp4_quantize(a_d, ga, sf_layout=nv.SF_LINEAR)
                asf = (asf_lin.view(torch.float8_e4m3fn).float().view(M, K // 16)
                       * (1.0 / ga)).contiguous()
            else:
                aq, asf, _ = nv.nvfp4_quantize(a_d, ga, sf_layout=layout_code)
            wq, wsf, _ = nv.nvfp4_quantize(w_d, gw, sf_layout=nv.SF_128x4)
            ops.append((aq, asf, wq, wsf))
        del a_d, w_d
        w_scale = (1.0 / gw).contiguous()
        out = torch.empty(M, N, dtype=torch.float16, device=dev)
        alg = algorithmic(wl, M=M, N=N, K=K, a_layout=args.a_layout)
        kernel_key = f"gemm_{wl}"
        kernel_name = {"decode": "gemm_nvfp4_decode_kernel<5,1>", "decode_f32": "gemm_nvfp4_decode_kernel<5,3>",
                       "prefill": "gemm_nvfp4_pair_kernel<4>"}.get(wl, "gemm_nvfp4_kernel")

        if wl == "decode_f32":
            ws_bytes = nv.nvfp4_gemm_act_f32_workspace_bytes(M, N, K)
        else:
            ws_bytes = nv.nvfp4_gemm_workspace_bytes(M, N, K)
        gemm_ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)  # zero on first use

        def gemm_call(aq, asf, wq, wsf, ws):
            if wl == "decode_f32":
                nv.nvfp4_gemm_act_f32(aq, asf, wq, wsf, w_scale, out=out, workspace=ws)
            else:
                nv.nvfp4_gemm(aq, asf, ga, wq, wsf, gw, a_layout=layout_code, out=out, workspace=ws)

        def step(i):
            gemm_call(*ops[i % ncopy], gemm_ws)
        launches_per_step, period = 1, ncopy
        if wl == "decode_f32":  # the scale-split kernel, then the GEMM, per 32 activation rows
            kernels_per_step = 2 * ((M + 31) // 32)
            launch_scope = ("the split kernel act_scale_planes_kernel<3> and the GEMM together "
                            "(one graph step; the GEMM alone is shorter)")
        workload_desc = workload_config(wl, args)
        assert (workload_desc["M"], workload_desc["N"], workload_desc["K"]) == (M, N, K)
        if wl in ("decode", "decode_f32"):
            unit, factor = "GB/s", alg["bytes"] / 1e9
        else:
            unit, factor = "TFLOP/s", alg["flops"] / 1e12
    else:
        raise SystemExit(f"unknown workload {wl}")

    torch.cuda.synchronize()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # The K timed steps are captured into one CUDA graph (the library calls are made while the
    # stream is captured: same kernels, same arguments, the inputs still rotated step by step),
    # the way a serving loop replays its kernels. Replaying it keeps host launch cost and the
    # per-graph launch latency (about 2 us per graph on B200) out of the device timing, which
    # matters for the tens-of-microsecond kernels; gaps between the kernels stay in.
    def run_steps(first, count):
        for i in range(count):
            step(first + i)
    if not args.no_graph:
        timed_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(timed_graph):
            for i in range(args.steps):
                step(args.warmup + i)
        torch.cuda.synchronize()
        timed_graph.replay()  # one untimed replay: the graph's first launch uploads it
        torch.cuda.synchronize()

        def run_steps(first, count):
            timed_graph.replay()

    # ---- timed region: K steps between two events on the launching stream. The step is one
    # launch of the path's kernel, so the kernel's average launch duration is the region's
    # time over K launches (gaps between launches included); events around each launch would
    # add their own gaps to short kernels.
    try:
        pr = torch.cuda.get_device_properties(dev)
        bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except Exception:
        bus = None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with Clocks(bus if rank == 0 else None) as clk:
        # Hold the stream in a short spin kernel (before the first event, so outside the timed
        # region) while the host enqueues the K steps: the region then starts with the first
        # step on the device instead of waiting for the host's launch.
        torch.cuda._sleep(max(1_000_000, 40_000 * args.steps))
        t0.record(stream)
        run_steps(args.warmup, args.steps)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    launch_avg = total_ms / (args.steps * launches_per_step)
    if kernels_per_step is None:
        kernels_per_step = launches_per_step
    total_ms = max_over_ranks(total_ms, dist, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, factor, ms_per_step)

    # ---- end to end through the public API with host buffers (pinned), copies timed
    e2e = None
    if wl in ("per_token", "swiglu", "swiglu_fp8"):
        src = copies[0]
        h_in = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
        h_in.copy_(src.cpu())
        h_q = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        h_sf = torch.empty(sf.shape, dtype=sf.dtype, pin_memory=True) if wl != "swiglu_fp8" else None
        h_g = torch.empty(g.shape, dtype=g.dtype, pin_memory=True) if wl == "per_token" else None
        d_in = torch.empty_like(src)

        def e2e_step():
            d_in.copy_(h_in, non_blocking=True)
            if wl == "per_token":
                nv.nvfp4_quantize(d_in, g, per_token=True, sf_layout=nv.SF_128x4, q=q, sf=sf)
                h_g.copy_(g, non_blocking=True)
            elif wl == "swiglu":
                nv.swiglu_nvfp4_quantize(d_in, gdev, sf_layout=nv.SF_128x4, q=q, sf=sf)
            else:
                nv.swiglu_fp8_quantize(d_in, sdev, q=q)
            h_q.copy_(q, non_blocking=True)
            if h_sf is not None:
                h_sf.copy_(sf, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist, dev)
        d2h = h_q.numel() + (h_sf.numel() if h_sf is not None else 0) + (h_g.numel() * 4 if h_g is not None else 0)
        e2e = {"value": job_throughput(world, factor, e2e_ms), "unit": unit,
               "h2d_bytes_per_step": h_in.numel() * 2, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms}
    elif wl in ("decode", "prefill", "tiny", "decode_f32"):
        aq, asf, wq, wsf = ops[0]
        hs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (aq, asf, wq, wsf)]
        for h, t in zip(hs, (aq, asf, wq, wsf)):
            h.copy_(t.cpu())
        ds = [torch.empty_like(t) for t in (aq, asf, wq, wsf)]
        h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

        def e2e_step():
            for d, h in zip(ds, hs):
                d.copy_(h, non_blocking=True)
            gemm_call(ds[0], ds[1], ds[2], ds[3], gemm_ws)
            h_out.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        n_e2e = 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist, dev)
        e2e = {"value": job_throughput(world, factor, e2e_ms), "unit": unit,
               "h2d_bytes_per_step": sum(h.numel() for h in hs), "d2h_bytes_per_step": h_out.numel() * 2,
               "ms_per_step": e2e_ms}

    # ---- roofline of the dominant kernel (the only kernel of the step)
    pk, pk_kind = peaks()
    if unit == "GB/s":
        achieved = alg["bytes"] / 1e9 / (launch_avg / 1e3)
        peak = float(pk["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": f"{pk_kind} hbm_gbs (copy)",
                "peak_nominal": NOMINAL_HBM_GBS, "frac_nominal": achieved / NOMINAL_HBM_GBS}
    else:
        achieved = alg["flops"] / 1e12 / (launch_avg / 1e3)
        peak = float(pk["bf16_tflops"]) * FP4_OVER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_source": f"{pk_kind} bf16_tflops (burst) x {FP4_OVER_BF16:g} nominal fp4/bf16 ratio",
                "peak_nominal": FP4_COUNTER_PEAK_TFLOPS,
                "frac_nominal": achieved / FP4_COUNTER_PEAK_TFLOPS}
    roof["traffic"] = recorded_traffic(kernel_key)
    roof["algorithmic_bytes_per_launch"] = alg["bytes"]
    roof["kernel"] = kernel_name
    roof["launch_ms"] = launch_avg
    if launch_scope is not None:
        roof["launch_ms_covers"] = launch_scope

    result = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {**workload_desc, "parallelism": f"replicas x{world}",
                   "timing": "direct calls" if args.no_graph else
                   "one CUDA graph holding the K timed steps (one library call each), replayed once"},
        "roofline": roof, "e2e": e2e, "gpu_launches": kernels_per_step * args.steps,
        "clocks": clk.summary() if rank == 0 else None,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, args)
    return result


# ----------------------------------------------------------------------------- oracle arm

def _oracle_sample(wl, args):
    """A bounded sample of the same workload for the oracle: returns (callable, units, desc)."""
    import numpy as np

    import oracle
    from nvfp4_block_scaled_10_b200 import workloads

    if wl == "per_token":
        rows = args.cpu_rows
        x = workloads.per_token(8192, 7168)
        bits = workloads.bits16(x[:rows])
        alg = algorithmic("per_token", M=rows, K=7168)
        return (lambda: oracle.quantize(bits, oracle.BF16, per_token=True)), alg["bytes"] / 1e9, \
            f"first {rows} of 8192 rows", "GB/s"
    if wl == "swiglu":
        rows = max(1, args.cpu_rows // 2)
        x = workloads.swiglu(rows, 14336)
        bits = workloads.bits16(x)
        g = 2688.0 / 60.0
        alg = algorithmic("swiglu", M=rows, H=14336)
        return (lambda: oracle.swiglu_quantize(bits, g, oracle.BF16)), alg["bytes"] / 1e9, \
            f"{rows} of 4096 rows", "GB/s"
    if wl == "swiglu_fp8":
        rows = max(1, args.cpu_rows // 2)
        x = workloads.swiglu(rows, 14336)
        bits = workloads.bits16(x)
        alg = algorithmic("swiglu_fp8", M=rows, H=14336)
        return (lambda: oracle.swiglu_fp8(bits, 448.0 / 60.0, oracle.BF16)), alg["bytes"] / 1e9, \
            f"{rows} of 4096 rows", "GB/s"
    if wl == "decode_f32":
        M, N, K = args.m, 512, 8192
        a, w = workloads.decode(args.m, 28672, 8192)
        ab, wb = workloads.bits16(a), workloads.bits16(w[:N])
        ga, gw = oracle.global_scale(ab), oracle.global_scale(workloads.bits16(w))
        aq, sa, _ = oracle.quantize(ab, g=ga)
        wq, sw, _ = oracle.quantize(wb, g=gw)
        table = np.array([oracle.e4m3_value(c) for c in range(256)], np.float64)
        sa32 = np.float32(table[sa] * np.float64(np.float32(1.0 / ga)))
        w_scale = float(np.float32(1.0 / gw))
        alg = algorithmic("decode_f32", M=M, N=N, K=K)
        return (lambda: oracle.gemm_act_f32(aq, sa32, wq, sw, w_scale)), alg["bytes"] / 1e9, \
            f"M={args.m}, 512 of 28672 weight rows", "GB/s"
    if wl in ("decode", "prefill", "tiny"):
        if wl == "decode":
            M, N, K = args.m, 512, 8192
            a, w = workloads.decode(args.m, 28672, 8192)
            w = w[:N]
            desc = f"M={args.m}, 512 of 28672 weight rows"
        elif wl == "prefill":
            M, N, K = 64, 1024, 8192
            a, w = workloads.prefill()
            a, w = a[:M], w[:N]
            desc = "64 of 8192 rows x 1024 of 8192 columns"
        else:
            a, w = workloads.tiny()
            M, K = a.shape
            N = w.shape[0]
            desc = "full"
        ab, wb = workloads.bits16(a), workloads.bits16(w)
        ga, gw = oracle.global_scale(ab), oracle.global_scale(wb)
        aq, sa, _ = oracle.quantize(ab, g=ga)
        wq, sw, _ = oracle.quantize(wb, g=gw)
        if wl == "decode":
            alg = algorithmic("decode", M=M, N=N, K=K)
            return (lambda: oracle.gemm(aq, sa, ga, wq, sw, gw)), alg["bytes"] / 1e9, desc, "GB/s"
        return (lambda: oracle.gemm(aq, sa, ga, wq, sw, gw)), 2 * M * N * K / 1e12, desc, "TFLOP/s"
    raise ValueError(wl)


def _threads_used():
    # the oracle is single-threaded C; numpy's fp64 matmul may use BLAS threads
    try:
        from threadpoolctl import threadpool_info
        n = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        n = 1
    return n


def _oracle_rows(wl):
    """The row-independent oracle workloads over all their rows: (run(lo, hi), rows, units
    of the whole sample, desc). The oracle's C calls release the GIL, so threads over row slices run it
    on all cores as it stands."""
    import oracle
    from nvfp4_block_scaled_10_b200 import workloads

    if wl == "per_token":
        bits = workloads.bits16(workloads.per_token(8192, 7168))
        return (lambda lo, hi: oracle.quantize(bits[lo:hi], oracle.BF16, per_token=True)), 8192, \
            algorithmic("per_token", M=8192, K=7168)["bytes"] / 1e9, "all 8192 rows"
    if wl in ("swiglu", "swiglu_fp8"):
        bits = workloads.bits16(workloads.swiglu(4096, 14336))
        if wl == "swiglu":
            run = lambda lo, hi: oracle.swiglu_quantize(bits[lo:hi], 2688.0 / 60.0, oracle.BF16)  # noqa: E731
        else:
            run = lambda lo, hi: oracle.swiglu_fp8(bits[lo:hi], 448.0 / 60.0, oracle.BF16)  # noqa: E731
        return run, 4096, algorithmic(wl, M=4096, H=14336)["bytes"] / 1e9, "all 4096 rows"
    return None


def _all_cores(wl):
    """The same oracle on every host core: row slices over one thread per core."""
    from concurrent.futures import ThreadPoolExecutor

    spec = _oracle_rows(wl)
    if spec is None:
        return None
    run, rows, units, desc = spec
    n = max(1, min(os.cpu_count() or 1, rows))
    cuts = [rows * i // n for i in range(n + 1)]
    t = time.perf_counter()
    with ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(lambda i: run(cuts[i], cuts[i + 1]), range(n)))
    dt = time.perf_counter() - t
    return {"value": units / dt, "cores": n, "sample": desc, "seconds": dt}


def cpu_baseline(wl, args):
    import oracle

    oracle.lib()  # build check and library load stay out of the timing
    fn, units, desc, unit = _oracle_sample(wl, args)
    # repeat the sample until about args.cpu_seconds of CPU work have run
    reps, t = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        dt = time.perf_counter() - t
        if dt >= args.cpu_seconds or reps >= 10000:
            break
    cores = 1 if wl in ("per_token", "swiglu", "swiglu_fp8") else _threads_used()
    out = {"value": units * reps / dt, "unit": unit, "cores": cores, "kind": "oracle",
           "sample": f"{desc}, {reps} run(s)", "seconds": dt}
    if not args.no_all_cores:
        allc = _all_cores(wl)
        if allc is not None:
            out["all_cores"] = allc
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return None
    fn, units, desc, unit = _oracle_sample(args.workload, args)
    for _ in range(args.warmup):
        fn()
    t = time.perf_counter()
    for _ in range(args.steps):
        fn()
    dt = (time.perf_counter() - t) / args.steps
    cores = 1 if args.workload in ("per_token", "swiglu", "swiglu_fp8") else _threads_used()
    value = units / dt
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {**workload_config(args.workload, args), "parallelism": f"replicas x{world}",
                       "sample": desc, "runs": "CPU oracle (plain C)"},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main

def sub_configs(args):
    """Workloads measured after the headline one (every rank runs the same list)."""
    if args.configs == "none":
        return []
    if args.configs == "auto":
        return list(DEFAULT_CONFIGS) if args.workload == "per_token" else []
    names = [c.strip() for c in args.configs.split(",") if c.strip()]
    for c in names:
        if c not in ("per_token", "swiglu", "swiglu_fp8", "decode", "decode_f32", "prefill", "tiny"):
            raise SystemExit(f"unknown workload in --configs: {c}")
    return [c for c in names if c != args.workload]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="per_token",
                    choices=["per_token", "swiglu", "swiglu_fp8", "decode", "decode_f32", "prefill",
                             "tiny"])
    ap.add_argument("--configs", default="auto",
                    help="comma-separated workloads measured after the headline one and reported "
                         "under 'configs' (decode at M=32, 128x4); 'auto' = prefill,decode when the "
                         "headline is the default per-token quantize, 'none' = no others")
    ap.add_argument("--m", type=int, default=32, help="tokens of the decode workload")
    ap.add_argument("--a-layout", default="128x4", choices=["128x4", "8x4"])
    ap.add_argument("--cpu-rows", type=int, default=2048)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="cpu_baseline repeats its oracle sample until this much time has run")
    ap.add_argument("--no-all-cores", action="store_true",
                    help="skip the oracle timing on all host cores (cpu_baseline.all_cores)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time direct library calls instead of CUDA-graph replays of them")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod

        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    try:
        res = run_ours(args, rank, world, torch, dist)
        subs = []
        for name in sub_configs(args):
            torch.cuda.empty_cache()
            sub_args = argparse.Namespace(**{**vars(args), "workload": name, "m": 32,
                                             "a_layout": "128x4"})
            r = run_ours(sub_args, rank, world, torch, dist)
            subs.append({k: v for k, v in r.items() if k not in ("metric", "n_gpus", "warmup",
                                                                  "higher_is_better", "scaling",
                                                                  "data", "dtype")})
        if subs:
            res["configs"] = subs
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
