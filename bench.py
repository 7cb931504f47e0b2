#!/usr/bin/env python
"""Benchmark of the Conv3D implicit-GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of the workload's
synthetic input: the convolution with fused NVFP4 activation fake-quant
(conv3d_implicit_gemm_pad2, quant_act as the workload says) followed by the
standalone fake-quantisation of the same activation tensor (fp4_fake_quant).
The metric is 2*M*Cout*K / step time in TFLOP/s (the convolution's
operations; the fake-quant adds time, not operations).  The default workload
is the largest single-GPU layer (the full-resolution 96-channel edge conv);
the same JSON line also carries a `layers` object with the convolution alone
timed on every workload.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronisation on both sides, measured with CUDA events on the
launching stream; the reported time is the maximum over ranks.  Inputs rotate
over enough copies that the working set exceeds the 126 MB L2, so no step
starts with its operands in L2.  SM clocks and throttle reasons are sampled
through NVML during the timed region.

Multi-GPU (torchrun): every rank runs its own independent copy of the layer
on its own seeded input (weak scaling, no collective on the data path);
value = all ranks' operations / max-over-ranks time.

--impl reference times the CPU oracle (the test infrastructure's plain
reference) on the host cores for the same workload, each step a bounded,
uniformly scaled-down sample of the step (a fraction f of the output rows
and the same fraction of the fake-quant elements); its value is the rate
measured on that sample, ms_per_step the measured sample time, and the
full-layer time it implies is reported separately as an estimate.  Only
rank 0 does work.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


KERNEL_SOURCES = ("conv3d_igemm_tmem.cu", "conv3d_igemm_tmem_sa.cu", "conv3d_tmem_kernel.cuh", "sm100_ptx.cuh",
                  "nvfp4.cuh")
# nominal dense FP4 : BF16 tensor throughput of B200 (9 : 2.25 PFLOP/s); the
# FP4 roofline is the measured BF16 peak times this ratio
FP4_OVER_BF16 = 4.0


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary of this workload, or None when there is none or the kernel
    sources have changed since it was captured (sha256 recorded beside it)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", f"conv3d_igemm_tmem_{workload}.md")
    try:
        with open(p) as f:
            text = f.read()
        h = hashlib.sha256()
        for name in KERNEL_SOURCES:
            with open(os.path.join(ROOT, "quantized_conv3d_implicit_b200", "csrc", name), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    fields = dict(line.split(":", 1) for line in text.splitlines()
                  if line.startswith(("source_sha256:", "traffic_bytes_per_launch:")))
    if fields.get("source_sha256", "").strip() != h.hexdigest():
        return None
    try:
        return int(fields["traffic_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clock sampling (NVML reads only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
            self.ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, b in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def pad6(wl):
    return (wl.pad_lo[0], wl.pad_hi[0], wl.pad_lo[1], wl.pad_hi[1], wl.pad_lo[2], wl.pad_hi[2])


def workload_config(wl, world: int = 1, fp4: bool = False) -> dict:
    """The `config` object of the JSON line (identical in both arms)."""
    od, oh, ow = wl.out_spatial()
    esz = {"torch.bfloat16": 2, "torch.float16": 2, "torch.float32": 4}[str(wl.dtype)]
    x_b = esz
    for d in wl.x_shape:
        x_b *= d
    y_b = esz * wl.x_shape[0] * wl.cout * od * oh * ow
    w_b = esz * wl.cout * wl.k_gemm
    set_mib = (x_b + w_b + y_b) / 2**20
    n_sets = max(2, -(-2 * L2_BYTES // (x_b + w_b + y_b)))
    return {
        "workload": wl.name, "x": list(wl.x_shape), "w": [wl.cout, wl.x_shape[1], *wl.kernel],
        "stride": list(wl.stride), "pad_lo": list(wl.pad_lo), "pad_hi": list(wl.pad_hi), "dil": list(wl.dil),
        "quant_act": wl.quant_act, "M": wl.m_gemm, "N": wl.cout, "K": wl.k_gemm, "out": [od, oh, ow],
        "step": ("conv3d_implicit_gemm_fp4 (weights packed beforehand) + fp4_fake_quant(x)" if fp4
                 else "conv3d_implicit_gemm(quant_act) + fp4_fake_quant(x)"),
        "l2": (f"x+w+y = {set_mib:.0f} MiB per input set; the GPU arm rotates {n_sets} sets "
               f"({n_sets * set_mib:.0f} MiB > 126 MiB L2)"),
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
    }


def make_sets(wl, dev, seed, with_fq: bool):
    """The workload's seeded inputs plus copies, so that the rotated working
    set exceeds twice the L2."""
    import torch

    from quantized_conv3d_implicit_b200 import workloads
    base = workloads.make_inputs(dataclass_replace(wl, seed=seed), device=dev, with_out=True)
    per_set = sum(t.numel() * t.element_size() for t in (base["x"], base["w"], base["out"]))
    n_sets = max(2, -(-2 * L2_BYTES // per_set))
    sets = [base] + [{k: (v.clone() if torch.is_tensor(v) else v) for k, v in base.items()} for _ in range(n_sets - 1)]
    if with_fq:
        for s in sets:
            s["fq"] = torch.empty_like(s["x"])
    return sets


def conv_call(api, wl, s, stream):
    if "wq" in s:   # the true-FP4 convolution over weights packed beforehand
        api.conv3d_implicit_gemm_fp4(s["x"], s["wq"], s["bias"], wl.stride, pad6(wl), wl.dil, s["act_amax"],
                                     out=s["out"], stream=stream)
        return
    api.conv3d_implicit_gemm(s["x"], s["w"], s["bias"], wl.stride, pad6(wl), wl.dil, s["act_amax"],
                             wl.quant_act, out=s["out"], stream=stream)


def time_conv_only(api, wl, sets, stream, dev, steps, warmup):
    """Mean and minimum device time (ms) of the convolution alone over
    `steps` launches rotating over the input sets, CUDA events on the
    launching stream, after `warmup` launches."""
    import torch
    for i in range(warmup):
        conv_call(api, wl, sets[i % len(sets)], stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i, (a, b) in enumerate(ev):
        a.record(stream)
        conv_call(api, wl, sets[i % len(sets)], stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    if api.check_device_error(stream) != 0:
        raise RuntimeError(f"device error in {wl.name}")
    t = [a.elapsed_time(b) for a, b in ev]
    return statistics.mean(t), min(t)


def time_fp4_only(api, wl, sets, stream, dev, steps, warmup):
    """As time_conv_only for the true-FP4 convolution (weights packed once per
    input set, outside the timed launches)."""
    import torch
    packed = [api.conv3d_fp4_pack_weights(s["w"], api.act_amax(s["w"], stream=stream), stream=stream) for s in sets]

    def call(i):
        s = sets[i % len(sets)]
        api.conv3d_implicit_gemm_fp4(s["x"], packed[i % len(sets)], s["bias"], wl.stride, pad6(wl), wl.dil,
                                     s["act_amax"], out=s["out"], stream=stream)
    for i in range(warmup):
        call(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i, (a, b) in enumerate(ev):
        a.record(stream)
        call(i)
        b.record(stream)
    torch.cuda.synchronize(dev)
    if api.check_device_error(stream) != 0:
        raise RuntimeError(f"device error in the FP4 convolution of {wl.name}")
    t = [a.elapsed_time(b) for a, b in ev]
    return statistics.mean(t), min(t)


def run_layers(api, args, stream, dev, peak, headline_sets, headline_name, rank):
    """Every workload's convolution alone: us, TFLOP/s and fraction of the
    measured BF16 peak, with the clocks seen while they ran; and (unless
    --no-fp4) the true-FP4 convolution of every quantised workload against
    the FP4 roofline (measured BF16 peak x FP4_OVER_BF16)."""
    import torch

    from quantized_conv3d_implicit_b200 import workloads
    steps = max(5, min(args.steps, 20))
    out, fp4 = {}, {}
    sampler = ClockSampler(dev.index)
    sampler.start()
    for name, wl in workloads.WORKLOADS.items():
        sets = headline_sets if name == headline_name else make_sets(wl, dev, wl.seed + 1000 * rank, False)
        mean_ms, min_ms = time_conv_only(api, wl, sets, stream, dev, steps, max(3, args.warmup))
        tf = wl.flops / (mean_ms * 1e-3) / 1e12
        out[name] = {"us": round(mean_ms * 1e3, 2), "us_min": round(min_ms * 1e3, 2), "tflops": round(tf, 2),
                     "frac": round(tf / peak, 4), "launches": steps}
        if not args.no_fp4 and wl.quant_act:
            f_ms, f_min = time_fp4_only(api, wl, sets, stream, dev, steps, max(3, args.warmup))
            ftf = wl.flops / (f_ms * 1e-3) / 1e12
            fp4[name] = {"us": round(f_ms * 1e3, 2), "us_min": round(f_min * 1e3, 2), "tflops": round(ftf, 2),
                         "frac": round(ftf / (peak * FP4_OVER_BF16), 4), "speedup_vs_bf16": round(mean_ms / f_ms, 3),
                         "launches": steps}
        if sets is not headline_sets:
            del sets
            torch.cuda.empty_cache()
    clocks = sampler.stop()
    return out, fp4, clocks


def run_ours(args, world, rank, local):
    import torch

    from quantized_conv3d_implicit_b200 import api, workloads

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    wl = workloads.get(args.workload)
    api.load_library()
    stream = torch.cuda.current_stream(dev)

    # independent seeded input per rank; rotate copies so the working set exceeds L2
    sets = make_sets(wl, dev, wl.seed + 1000 * rank, True)
    n_sets = len(sets)
    fp4 = args.conv == "fp4"
    if fp4:   # weights packed once per set, before the timed region
        for s_ in sets:
            s_["wq"] = api.conv3d_fp4_pack_weights(s_["w"], api.act_amax(s_["w"], stream=stream), stream=stream)
    base = sets[0]

    def step(s):
        conv_call(api, wl, s, stream)
        api.fp4_fake_quant(s["x"], s["act_amax"], out=s["fq"], stream=stream)

    for i in range(args.warmup):
        step(sets[i % n_sets])
    torch.cuda.synchronize(dev)
    if api.check_device_error(stream) != 0:
        raise RuntimeError("device error during warm-up")

    # timed region: K steps; per-kernel events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    sampler.start()
    t0.record(stream)
    for i in range(args.steps):
        s = sets[i % n_sets]
        a, b, c = ev[i]
        a.record(stream)
        conv_call(api, wl, s, stream)
        b.record(stream)
        api.fp4_fake_quant(s["x"], s["act_amax"], out=s["fq"], stream=stream)
        c.record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world, dev)
    local_ms = t0.elapsed_time(t1)
    conv_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    fq_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    if api.check_device_error(stream) != 0:
        raise RuntimeError("device error during timing")
    total_ms = max_over_ranks(local_ms, world, dev)
    ms_per_step = total_ms / args.steps
    tflops = world * wl.flops * args.steps / (total_ms * 1e-3) / 1e12

    peaks, peaks_src = load_peaks()
    peak = peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    x_bytes = base["x"].numel() * base["x"].element_size()

    # the global amax that feeds the quantiser (device reduction, outside the
    # step): L2 flushed before every launch, so x streams from HBM
    amax_us = time_act_amax(base["x"], stream, dev, args.steps)

    # every workload's convolution alone (outside the step's timed region)
    layers, layers_fp4, layer_clocks = (None, None, None)
    if fp4:
        for s_ in sets:
            del s_["wq"]
    if not args.no_layers:
        layers, layers_fp4, layer_clocks = run_layers(api, args, stream, dev, peak, sets, wl.name, rank)

    formats = None if (args.no_formats or fp4) else time_formats(api, wl, base, stream, dev, hbm, peak)

    # context only: the same convolutions without quantisation in cuDNN
    cudnn = None if (args.no_cudnn or fp4) else time_cudnn(dev, peak, layers)

    # end-to-end through the public API with pinned host buffers
    e2e = None if (args.no_e2e or fp4) else run_e2e(args, wl, base, stream, dev, world)

    conv_tflops = wl.flops / (conv_ms * 1e-3) / 1e12
    conv_peak = peak * (FP4_OVER_BF16 if fp4 else 1.0)
    launches_per_step = 2 + (0 if (wl.dtype == torch.bfloat16 and wl.k_gemm % 8 == 0) else 1)
    fq_bytes = 2 * x_bytes  # read x, write the fake-quantised copy
    result = {
        "metric": "Conv3D TFLOP/s (2*M*N*K) and % of B200 BF16 dense peak; us/layer",
        "value": round(tflops, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[wl.dtype]
                 + ("->nvfp4 mma (kind::mxf4nvf4), f32 acc" if fp4 else "->bf16 mma, f32 acc"),
        "data": "synthetic (seeded N(0,1) activations, N(0,1/sqrt(K)) weights)",
        "config": workload_config(wl, world, fp4),
        "layer_us": round(conv_ms * 1e3, 2),
        "fake_quant_us": round(fq_ms * 1e3, 2),
        "layer_frac_of_peak": round(conv_tflops / conv_peak, 4),
        "roofline": {
            "bound": "tensor", "achieved": round(conv_tflops, 2), "peak": round(conv_peak, 1), "unit": "TFLOP/s",
            "frac": round(conv_tflops / conv_peak, 4), "traffic": None if fp4 else profiled_traffic(wl.name),
            "kernel": "conv3d_igemm_tmem, NVFP4 operands (dominant)" if fp4 else "conv3d_igemm_tmem (dominant)",
            "peak_source": (f"{peaks_src} bf16_tflops (burst) x {FP4_OVER_BF16:g} (nominal FP4:BF16 dense ratio)"
                            if fp4 else f"{peaks_src} bf16_tflops (burst)"),
        },
        "fake_quant": {
            "us": round(fq_ms * 1e3, 2), "bytes": fq_bytes, "bound": "hbm",
            "achieved": round(fq_bytes / (fq_ms * 1e-3) / 1e9, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(fq_bytes / (fq_ms * 1e-3) / 1e9 / hbm, 4), "kernel": "fp4_fake_quant_kernel",
            "l2": "timed inside the step (inputs rotate past L2)", "peak_source": f"{peaks_src} hbm_gbs",
        },
        "act_amax": {
            "us": round(amax_us, 2), "bytes": x_bytes, "bound": "hbm",
            "achieved": round(x_bytes / (amax_us * 1e-6) / 1e9, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(x_bytes / (amax_us * 1e-6) / 1e9 / hbm, 4),
            "kernel": "act_amax_kernel", "l2": "flushed (256 MiB write) before each launch",
            "peak_source": f"{peaks_src} hbm_gbs",
        },
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
    }
    if layers is not None:
        result["layers"] = layers
        result["layers_clocks"] = layer_clocks
    if formats is not None:
        result["formats"] = formats
    if cudnn is not None:
        result["cudnn_context"] = cudnn
    if layers_fp4:
        result["layers_fp4"] = {
            "what": ("conv3d_implicit_gemm_fp4: activations and weights NVFP4, block-scaled FP4 MMA "
                     "(kind::mxf4nvf4), weights packed outside the timed launches"),
            "peak": round(peak * FP4_OVER_BF16, 1), "unit": "TFLOP/s",
            "peak_source": f"{peaks_src} bf16_tflops (burst) x {FP4_OVER_BF16:g} (nominal FP4:BF16 dense ratio)",
            "layers": layers_fp4,
        }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, base, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def dataclass_replace(wl, **kw):
    import dataclasses
    return dataclasses.replace(wl, **kw)


def run_e2e(args, wl, base, stream, dev, world):
    """Same metric through the public calls with pinned host inputs: every step
    copies x, w, bias and act_amax host->device, runs the hot path and copies
    the convolution output and the fake-quantised tensor back.  Steps are
    pipelined over two device buffer sets and three streams (copy-in,
    compute, copy-out), as a serving loop would run them: step i's inputs
    travel while step i-1 computes and step i-2's results travel back; every
    step's own copies stay inside the timed region."""
    import torch

    from quantized_conv3d_implicit_b200 import api

    host = {k: (v.cpu().pin_memory() if torch.is_tensor(v) else v) for k, v in base.items()
            if k in ("x", "w", "bias", "act_amax")}
    bufs = []
    for _ in range(2):
        bufs.append({"x": torch.empty_like(base["x"]), "w": torch.empty_like(base["w"]),
                     "b": None if base["bias"] is None else torch.empty_like(base["bias"]),
                     "a": torch.empty_like(base["act_amax"]), "y": torch.empty_like(base["out"]),
                     "q": torch.empty_like(base["x"])})
    hy = torch.empty(base["out"].shape, dtype=base["out"].dtype, pin_memory=True)
    hq = torch.empty(base["x"].shape, dtype=base["x"].dtype, pin_memory=True)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_c = stream
    # per buffer set: its inputs have landed / its compute is done / its results have left
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def step(i):
        b = bufs[i % 2]
        k = i % 2
        if used[k]:
            s_in.wait_event(ev_c[k])      # the set's previous compute has read its inputs
        with torch.cuda.stream(s_in):
            b["x"].copy_(host["x"], non_blocking=True)
            b["w"].copy_(host["w"], non_blocking=True)
            if b["b"] is not None:
                b["b"].copy_(host["bias"], non_blocking=True)
            b["a"].copy_(host["act_amax"], non_blocking=True)
        ev_in[k].record(s_in)
        s_c.wait_event(ev_in[k])
        if used[k]:
            s_c.wait_event(ev_out[k])     # the set's previous results have been copied out
        api.conv3d_implicit_gemm(b["x"], b["w"], b["b"], wl.stride, pad6(wl), wl.dil, b["a"], wl.quant_act,
                                 out=b["y"], stream=s_c)
        api.fp4_fake_quant(b["x"], b["a"], out=b["q"], stream=s_c)
        ev_c[k].record(s_c)
        s_out.wait_event(ev_c[k])
        with torch.cuda.stream(s_out):
            hy.copy_(b["y"], non_blocking=True)
            hq.copy_(b["q"], non_blocking=True)
        ev_out[k].record(s_out)
        used[k] = True

    steps = max(3, min(args.steps, 20))
    for i in range(2):
        step(i)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    t0.record(s_in)
    for i in range(2, 2 + steps):
        step(i)
    s_out.wait_event(ev_c[(1 + steps) % 2])
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / steps
    h2d = sum(t.numel() * t.element_size() for t in (host["x"], host["w"], host["act_amax"])) + \
        (0 if base["bias"] is None else base["bias"].numel() * base["bias"].element_size())
    d2h = hy.numel() * hy.element_size() + hq.numel() * hq.element_size()
    return {"value": round(world * wl.flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "pipelined": "2 buffer sets, copy-in / compute / copy-out streams"}


# ---------------------------------------------------------------------------
# CPU oracle timing (test infrastructure: the only place bench.py runs it)
# ---------------------------------------------------------------------------

def oracle_sample_step(wl, x_np, w_np, b_np, amax, rows, rng, w_amax=None):
    """One scaled-down step on the host cores: `rows` random output rows (all
    Cout) of the convolution and the same fraction rows / M of the
    fake-quant elements (whole blocks).  With w_amax, the convolution is the
    true-FP4 one (both operands NVFP4).  Returns (conv s, fake-quant s,
    fraction of the step done)."""
    import oracle
    ms = rng.integers(0, wl.m_gemm, rows)
    t = time.perf_counter()
    if w_amax is not None:
        oracle.conv3d_nvfp4(x_np, w_np, b_np, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil, act_amax=amax, w_amax=w_amax,
                            m_list=ms)
    else:
        oracle.conv3d(x_np, w_np, b_np, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil, wl.quant_act, amax, m_list=ms)
    t_conv = time.perf_counter() - t
    frac = rows / wl.m_gemm
    fq_elems = max(16, int(round(x_np.size * frac / 16)) * 16)
    start = int(rng.integers(0, max(1, (x_np.size - fq_elems) // 16 + 1))) * 16
    t = time.perf_counter()
    oracle.fp4_fake_quant(x_np.reshape(-1)[start:start + fq_elems], amax)
    t_fq = time.perf_counter() - t
    return t_conv, t_fq, frac


def _rows_for(wl, x_np, w_np, b_np, amax, rng, seconds):
    t_conv, _, _ = oracle_sample_step(wl, x_np, w_np, b_np, amax, 16, rng)
    return int(max(32, min(wl.m_gemm, seconds / max(t_conv / 16, 1e-6))))


def cpu_baseline(wl, base, budget_s: float = 15.0):
    x_np = base["x"].float().cpu().numpy()
    w_np = base["w"].float().cpu().numpy()
    b_np = None if base["bias"] is None else base["bias"].float().cpu().numpy()
    amax = float(base["act_amax"].item())
    import numpy as np
    rng = np.random.default_rng(1234)
    rows = _rows_for(wl, x_np, w_np, b_np, amax, rng, budget_s * 0.8)
    t_conv, t_fq, frac = oracle_sample_step(wl, x_np, w_np, b_np, amax, rows, rng)
    sample_s = t_conv + t_fq
    return {"value": frac * wl.flops / sample_s / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{rows} random output rows x all {wl.cout} channels ({t_conv:.1f} s) + the same fraction "
                      f"({frac:.2e}) of the fake-quant elements ({t_fq:.2f} s); full layer would take "
                      f"about {sample_s / frac:.0f} s at this rate"}


def run_reference(args, world, rank, local):
    """The oracle on the host cores, same workload/metric; rank 0 only."""
    if rank != 0:
        return
    import numpy as np

    from quantized_conv3d_implicit_b200 import workloads
    wl = workloads.get(args.workload)
    base = workloads.make_inputs(wl, device="cpu")
    x_np = base["x"].float().numpy()
    w_np = base["w"].float().numpy()
    b_np = None if base["bias"] is None else base["bias"].float().numpy()
    amax = float(base["act_amax"].item())
    fp4 = args.conv == "fp4"
    w_amax = float(np.abs(w_np).max()) if fp4 else None
    rng = np.random.default_rng(99)
    rows = _rows_for(wl, x_np, w_np, b_np, amax, rng, 1.0)   # about 1 s of work per step
    for _ in range(args.warmup):
        oracle_sample_step(wl, x_np, w_np, b_np, amax, max(8, rows // 8), rng, w_amax)
    tot = 0.0
    frac = rows / wl.m_gemm
    for _ in range(args.steps):
        tc, tf, frac = oracle_sample_step(wl, x_np, w_np, b_np, amax, rows, rng, w_amax)
        tot += tc + tf
    step_s = tot / args.steps
    value = frac * wl.flops / step_s / 1e12
    sample = (f"each step: {rows} random output rows x all {wl.cout} channels + the same fraction ({frac:.2e}) "
              f"of the fake-quant elements")
    print(json.dumps({
        "impl": "reference",
        "metric": "Conv3D TFLOP/s (2*M*N*K) and % of B200 BF16 dense peak; us/layer",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 accumulate over bf16/fp4 operands (CPU oracle)", "data": "synthetic",
        "config": workload_config(wl, world, fp4),
        "sample_fraction": frac,
        "full_layer_ms_estimate": step_s / frac * 1e3,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def time_formats(api, wl, base, stream, dev, hbm, bf16_peak):
    """The quantiser formats beyond the article's default: the standalone
    NVFP4 fake-quant with blocks of 32..256 and MXFP4 (dequantised values,
    scale bytes and packed codes) on the layer's x, against the HBM roofline
    (L2 flushed before each launch); and the fused convolution with each
    format on the wan_mid layer (the tensor-memory kernel runs NVFP4 blocks
    of 16, 32 and 64 and MXFP4, the general kernel blocks of 128 and 256),
    against the BF16 peak."""
    import torch

    from quantized_conv3d_implicit_b200 import workloads
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    x, amax = base["x"], base["act_amax"]
    esz = x.element_size()
    n = x.numel()

    def timed(fn, reps=5):
        for _ in range(2):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b) * 1e3)
        if api.check_device_error(stream) != 0:
            raise RuntimeError("device error in a format timing")
        return statistics.mean(ts)

    out = {"x": wl.name, "standalone": {}, "fused_conv": {}}
    q = torch.empty_like(x)
    for bs in (32, 64, 128, 256):
        us = timed(lambda: api.fp4_fake_quant(x, amax, out=q, stream=stream, block_size=bs))
        by = 2 * n * esz
        out["standalone"][f"nvfp4_{bs}"] = {"us": round(us, 1), "gbs": round(by / (us * 1e-6) / 1e9, 1),
                                           "frac_hbm": round(by / (us * 1e-6) / 1e9 / hbm, 4)}
    scales = torch.empty(n // 32, dtype=torch.uint8, device=dev)
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    xs, os_ = api._tensor(x), api._tensor(q)
    lib = api.load_library()

    def mx():
        api._check(lib, lib.mxfp4_quantize(api._ref(xs), 0.0, api._ref(os_), scales.data_ptr(), codes.data_ptr(),
                                           api._stream_handle(stream)))
    us = timed(mx)
    by = n * esz + n * esz + n // 32 + n // 2
    out["standalone"]["mxfp4"] = {"us": round(us, 1), "gbs": round(by / (us * 1e-6) / 1e9, 1),
                                  "frac_hbm": round(by / (us * 1e-6) / 1e9 / hbm, 4)}
    del q, scales, codes
    torch.cuda.empty_cache()
    cw = workloads.get("wan_mid_384_bf16")
    inp = workloads.make_inputs(cw, device=dev, with_out=True)
    for fmt, bs, dst in (("nvfp4", 16, 0.0), ("nvfp4", 32, 0.0), ("nvfp4", 64, 0.0), ("nvfp4", 128, 0.0),
                         ("mxfp4", 32, 0.0)):
        us = timed(lambda: api.conv3d_implicit_gemm_ex(inp["x"], inp["w"], inp["bias"], cw.stride, pad6(cw), cw.dil,
                                                        inp["act_amax"], quant_format=fmt, block_size=bs,
                                                        dst_type_max=dst, out=inp["out"], stream=stream), reps=3)
        tf = cw.flops / (us * 1e-6) / 1e12
        out["fused_conv"][f"{fmt}_{bs}"] = {"layer": cw.name, "us": round(us, 1), "tflops": round(tf, 1),
                                           "frac": round(tf / bf16_peak, 4)}
    return out


def time_cudnn(dev, bf16_peak, layers):
    """Context, not a baseline of the method: torch's cuDNN convolution
    (F.conv3d, autotuned) on the Wan and edge layers without quantisation
    (cuDNN has no fused activation quantiser), the input padded outside the
    timed launches (the causal temporal padding is asymmetric), L2 flushed
    before each launch, CUDA events on the launching stream."""
    import torch
    import torch.nn.functional as F

    from quantized_conv3d_implicit_b200 import workloads
    torch.backends.cudnn.benchmark = True
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    cur = torch.cuda.current_stream(dev)
    out = {"what": "torch.nn.functional.conv3d (cuDNN), no quantisation; ours: this library with quantisation on "
                   "(and off where a quant-off workload exists)", "layers": {}}
    for name in ("wan_mid_384_bf16", "wan_hi_192_bf16", "edge_full_96_bf16"):
        cw = workloads.get(name)
        inp = workloads.make_inputs(cw, device=dev)
        xp = F.pad(inp["x"], (cw.pad_lo[2], cw.pad_hi[2], cw.pad_lo[1], cw.pad_hi[1], cw.pad_lo[0], cw.pad_hi[0]))
        del inp["x"]
        fn = lambda: F.conv3d(xp, inp["w"], inp["bias"], stride=cw.stride, dilation=cw.dil)  # noqa: E731
        for _ in range(3):
            y = fn()
        ts = []
        for _ in range(5):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(cur)
            y = fn()
            b.record(cur)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b) * 1e3)
        del y, xp, inp
        torch.cuda.empty_cache()
        us = statistics.median(ts)
        tf = cw.flops / (us * 1e-6) / 1e12
        row = {"us": round(us, 1), "tflops": round(tf, 1), "frac": round(tf / bf16_peak, 4)}
        if layers and name in layers:
            row["ours_quant_on_us"] = layers[name]["us"]
        if layers and name + "_noquant" in layers:
            row["ours_quant_off_us"] = layers[name + "_noquant"]["us"]
        out["layers"][name] = row
    return out


def time_act_amax(x, stream, dev, steps):
    """Mean device time (us) of q3d_act_amax on x (memset of the output word
    + one kernel), CUDA events on the launching stream, L2 flushed before
    each launch."""
    import torch

    from quantized_conv3d_implicit_b200 import api
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = torch.empty(1, dtype=torch.float32, device=dev)
    n = max(10, min(steps, 100))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for _ in range(3):
        api.act_amax(x, out=out, stream=stream)
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        api.act_amax(x, out=out, stream=stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    if api.check_device_error(stream) != 0:
        raise RuntimeError("device error in act_amax")
    return statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3


def main(argv=None):
    from quantized_conv3d_implicit_b200 import workloads
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=workloads.HEADLINE, choices=sorted(workloads.WORKLOADS) + sorted(workloads.CROPS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-layers", action="store_true", help="skip the per-workload convolution timings")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end timing with host copies")
    ap.add_argument("--no-fp4", action="store_true", help="skip the true-FP4 convolution timings")
    ap.add_argument("--no-formats", action="store_true", help="skip the other quantiser formats' timings")
    ap.add_argument("--no-cudnn", action="store_true", help="skip the cuDNN context timings")
    ap.add_argument("--conv", default="bf16", choices=["bf16", "fp4"],
                    help="the step's convolution: the fake-quantised BF16 path (default) or the true-FP4 variant")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        run_reference(args, world, rank, local)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
