#!/usr/bin/env python
"""Benchmark of the fully-integer attention forward on B200.

One step = one IntAttention forward (int8 Q.K^T -> IndexSoftmax -> u8 x s8
P.V -> int8) over one batch of the workload, through the C ABI.  Default
workload: the largest one, a LLaMA-7B-shaped causal prefill, B=1 H=32
L=8192 d=128.  The other prefill workloads (BERT-base L128 and B8 L512,
ViT-B/16 L197, GPT-2-small causal L2048) are timed the same way and reported
in the "prefill_configs" object of the same line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle, timed on host cores

Rank 0 prints one JSON line.  Timing: CUDA events on the launching stream,
max over ranks; inputs rotate over enough copies to exceed the 126 MB L2.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "IntAttention fwd effective int8 TOPS & % of INT8 tensor roofline; decode GB/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio: 4.5 POPS int8 / 2.25 PFLOP/s bf16


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="llama7b_causal_l8192")
    p.add_argument("--no-configs", action="store_true", help="skip the other prefill workloads")
    p.add_argument("--decode-workload", default="llama7b_decode_b64_lk4096")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--leg", choices=["decode", "decode_int4", "quantize", "gelu", "forward_fp", "calibrate"], default=None,
                   help="run only this secondary leg and print its object (for profiler captures)")
    return p.parse_args(argv)


# ------------------------------------------------------------ distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of x over all ranks (the slowest rank sets the time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_value(per_rank_units: float, world: int, seconds: float) -> float:
    """Whole-job throughput: units every rank processed / the max-over-ranks time."""
    return per_rank_units * world / seconds


# ------------------------------------------------------------------ peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(kernel: str, workload: str, key: str = "bytes_per_launch"):
    """DRAM bytes per launch (or per call) from a committed ncu summary, only
    while the kernel source still has the hash the counters were taken with."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(kernel, {}).get(workload)
    if not ent:
        return None
    h = hashlib.sha256()
    for rel in ent.get("sources", []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != ent.get("source_hash"):
        return None
    return ent.get(key)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and throttle reasons of one GPU, polled through NVML
    from a background thread every millisecond while the timed region runs
    (nvidia-smi's 200 ms period would miss a region of a few milliseconds)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._stop = None
        self._thread = None

    def _handle(self, pynvml):
        """NVML handle of the CUDA device (matched by PCI bus id, since NVML
        indices ignore CUDA_VISIBLE_DEVICES)."""
        try:
            import torch
            p = torch.cuda.get_device_properties(self.gpu)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:  # noqa: BLE001
            return pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = self._handle(pynvml)
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - no NVML: report no clocks
            return
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM)
                    pw = pynvml.nvmlDeviceGetPowerUsage(handle) / 1000.0
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                    self.samples.append((sm, pw, rs))
                except Exception:  # noqa: BLE001
                    pass
                time.sleep(0.001)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            return None
        sm = [s[0] for s in self.samples]
        pw = [s[1] for s in self.samples]
        reasons = sorted({n for s in self.samples for n, bit in self.REASONS.items() if s[2] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.sm_max,
                "power_w_max": round(max(pw), 1), "samples": len(sm), "reasons": reasons,
                "source": "NVML, 1 ms polling during the timed region"}


# ------------------------------------------------------------- our arm
PREFILL_WORKLOADS = ["bert_base_l128", "bert_base_b8_l512", "vit_b16_l197", "gpt2_small_causal_l2048",
                     "llama7b_causal_l8192"]


def rotation(w):
    """Number of input copies the timed steps rotate over (q, k, v, out of
    one step: their total exceeds the 126 MB L2 at least twice) and the bytes
    of one copy."""
    set_bytes = 2 * w.B * w.H * w.Lq * w.d + 2 * w.B * w.H * w.Lk * w.d
    return max(2, min(1024, math.ceil(2 * L2_BYTES / set_bytes))), set_bytes


def workload_config(w, world: int) -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    nsets, set_bytes = rotation(w)
    return {"workload": w.name, "B": w.B, "H": w.H, "Lq": w.Lq, "Lk": w.Lk, "d": w.d,
            "causal": w.causal, "clip_c": w.clip_c,
            "quant": "per_head" if w.per_head else "per_tensor",
            "l2": f"inputs rotate over {nsets} copies ({nsets * set_bytes / 2**20:.0f} MiB > 126 MiB L2)",
            "timing": "K steps captured as one CUDA graph, replayed once between CUDA events",
            "parallelism": f"dp{world} (independent problems)"}


def time_prefill(ia, w, x, dev, stream, steps: int, warmup: int, clocks=None, world: int = 1, variant: int = 0,
                 scales=None):
    """ms per forward of workload w: `steps` calls over rotating copies of the
    inputs, captured as one CUDA graph and replayed between CUDA events on
    `stream`; max over ranks."""
    import torch
    sc = scales if scales is not None else ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    nsets, _ = rotation(w)
    q0, k0, v0 = (torch.from_numpy(a).to(dev) for a in (x.q, x.k, x.v))
    sets = [(q0.clone(), k0.clone(), v0.clone(), torch.empty_like(q0)) for _ in range(nsets)]
    del q0, k0, v0

    def step(i):
        q, k, v, o = sets[i % nsets]
        ia.forward(q, k, v, sc, w.causal, w.clip_c, out=o, stream=stream, variant=variant)

    # everything on `stream`: the calls, the capture, the replay and the events
    # (the copies above ran on the default stream: complete them first)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            step(i)
        torch.cuda.synchronize(dev)
        if ia.device_error(stream) != ia.OK:
            raise RuntimeError("a kernel wait timed out during warm-up")
        # the timed steps are captured once as a CUDA graph and replayed: the
        # device time then excludes the host's per-call launch latency
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(steps):
                step(i)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        if clocks is not None:
            clocks.start()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    clk = clocks.stop() if clocks is not None else None
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    if ia.device_error(stream) != ia.OK:
        raise RuntimeError("a kernel wait timed out during the timed steps")
    del graph, sets
    return ms, clk


def _int8_peak(peaks, sustained: bool):
    key = "bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    return peaks[key] * INT8_OVER_BF16, key


def run_leg(args):
    """One secondary leg alone: its device footprint is its own inputs only."""
    import torch
    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    init_dist(world, "nccl")
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    if args.leg == "decode":
        out = run_decode(args, dev, stream, world, peaks, peak_src, args.decode_workload)
    elif args.leg == "decode_int4":
        out = run_decode(args, dev, stream, world, peaks, peak_src, "llama7b_decode_int4_b64_lk4096")
    elif args.leg == "quantize":
        out = run_quantize(args, dev, stream, world, peaks, peak_src)
    elif args.leg == "forward_fp":
        out = run_forward_fp(args, dev, stream, world, peaks, peak_src)
    elif args.leg == "calibrate":
        out = run_calibrate(args, dev, stream, world)
    else:
        out = run_gelu(args, dev, stream, world, peaks, peak_src)
    if rank == 0:
        print(json.dumps({"leg": args.leg, **out}), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_ours(args):
    import numpy as np
    import torch

    import integer_only_quantized_b200 as ia
    from integer_only_quantized_b200 import workloads as wl

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    init_dist(world, "nccl")
    w = wl.WORKLOADS[args.workload]
    assert not w.decode, "the headline workload is a prefill workload"
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    stream = torch.cuda.Stream(dev)
    clocks = ClockSampler(local_rank)
    ms, clk = time_prefill(ia, w, x, dev, stream, args.steps, args.warmup, clocks, world)
    ops = w.effective_ops
    value = aggregate_value(ops, world, ms * 1e-3) / 1e12

    # end to end through the public API with pinned HOST buffers: the
    # host-buffer forward copies q, k, v in and the output out every step,
    # pipelined in chunks over its copy streams and `stream`
    hq, hk, hv = (torch.from_numpy(a).pin_memory() for a in (x.q, x.k, x.v))
    ho = torch.empty(x.q.shape, dtype=torch.int8).pin_memory()
    hws = torch.empty(ia.forward_host_workspace_size(w.B, w.H, w.Lq, w.Lk, w.d), dtype=torch.uint8, device=dev)

    def e2e_step(i):
        ia.forward_host(hq, hk, hv, sc, w.causal, w.clip_c, out=ho, workspace=hws, stream=stream, device=dev)

    torch.cuda.synchronize(dev)  # inputs made on the default stream are complete before `stream` reads them
    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    err = ia.device_error(stream)
    if err != ia.OK:
        raise RuntimeError(f"device error {err} ({ia.strerror(err)}) in the host-buffer forward")
    e2e_val = aggregate_value(ops, world, e2e_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    peak_int8, peak_key = _int8_peak(peaks, sustained=False)
    achieved = ops / (ms * 1e-3) / 1e12  # one launch per step: per-launch duration = ms
    if achieved > 1.5 * peak_int8:
        raise RuntimeError(f"{achieved:.0f} TOPS is far above the int8 peak: the timed region missed the work")
    traffic = kernel_traffic("prefill_kernel", w.name)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": workload_config(w, world),
        "roofline": {"bound": "tensor", "kernel": "prefill_kernel", "achieved": round(achieved, 3),
                     "peak": round(peak_int8, 1), "unit": "TOPS", "frac": round(achieved / peak_int8, 4),
                     "peak_source": f"{peak_src} {peak_key} x {INT8_OVER_BF16} (dense int8/bf16)",
                     "traffic": traffic},
        "e2e": {"value": round(e2e_val, 3), "unit": "TOPS",
                "h2d_bytes_per_step": int(x.q.nbytes + x.k.nbytes + x.v.nbytes),
                "d2h_bytes_per_step": int(x.q.nbytes), "ms_per_step": round(e2e_ms, 5),
                "api": "intattn_forward_host (pinned host buffers; consecutive calls overlap through two workspace slots)"},
        "gpu_launches": args.steps,
        "clocks": clk,
    }

    if not args.no_configs:
        line["prefill_configs"] = run_prefill_configs(args, ia, dev, stream, world, peak_int8, w.name)
        line["zero_points"] = run_zero_point(args, ia, dev, stream, world, peak_int8, ms)
    if not args.no_decode:
        line["decode"] = run_decode(args, dev, stream, world, peaks, peak_src, args.decode_workload)
        line["decode_int4"] = run_decode(args, dev, stream, world, peaks, peak_src,
                                         "llama7b_decode_int4_b64_lk4096")
        line["quantize"] = run_quantize(args, dev, stream, world, peaks, peak_src)
        line["forward_fp"] = run_forward_fp(args, dev, stream, world, peaks, peak_src)
        line["calibrate"] = run_calibrate(args, dev, stream, world)
        line["gelu"] = run_gelu(args, dev, stream, world, peaks, peak_src)
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, x, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_prefill_configs(args, ia, dev, stream, world, peak_int8, skip):
    """Every other prefill workload, timed like the headline (rotating
    inputs, one CUDA graph of calls between CUDA events)."""
    from integer_only_quantized_b200 import workloads as wl
    res = {}
    for name in PREFILL_WORKLOADS:
        if name == skip:
            continue
        w = wl.WORKLOADS[name]
        x = wl.make_inputs(w)
        nsets, set_bytes = rotation(w)
        steps = max(args.steps, 100, nsets)  # every copy is used at least once
        ms, _ = time_prefill(ia, w, x, dev, stream, steps, max(3, args.warmup), None, world)
        tops = w.effective_ops / (ms * 1e-3) / 1e12
        # the kernel intattn_forward picks for this row length
        kname = "prefill_short_kernel" if w.Lk <= ia.SHORT_ROWS_MAX_KEYS else "prefill_kernel"
        if tops > 1.5 * peak_int8:
            raise RuntimeError(f"{name}: {tops:.0f} TOPS is far above the int8 peak: the timed region missed the work")
        res[name] = {"value": round(aggregate_value(w.effective_ops, world, ms * 1e-3) / 1e12, 3), "unit": "TOPS",
                     "ms_per_call": round(ms, 5), "calls": steps, "launches_per_call": 1,
                     "effective_ops": w.effective_ops,
                     "roofline": {"bound": "tensor", "achieved": round(tops, 3), "peak": round(peak_int8, 1),
                                  "unit": "TOPS", "frac": round(tops / peak_int8, 4),
                                  "kernel": kname, "traffic": kernel_traffic(kname, name)},
                     "l2": f"inputs rotate over {nsets} copies ({nsets * set_bytes / 2**20:.0f} MiB > 126 MiB L2)"}
        if w.Lk <= 2 * ia.SHORT_ROWS_MAX_KEYS:
            # both ways of handling a short row's scores on the same workload:
            # resident in tensor memory (what intattn_forward runs up to 256
            # keys) and recomputed per sweep (the three-pass kernel)
            variants = {}
            pairs = [("three_pass", ia.VARIANT_THREE_PASS)]
            if w.Lk <= ia.SHORT_ROWS_MAX_KEYS:
                pairs.insert(0, ("short_rows", ia.VARIANT_SHORT_ROWS))
            for vname, vid in pairs:
                vms, _ = time_prefill(ia, w, x, dev, stream, steps, max(3, args.warmup), None, world, vid)
                vt = w.effective_ops / (vms * 1e-3) / 1e12
                variants[vname] = {"ms_per_call": round(vms, 5), "value": round(vt, 3),
                                   "frac": round(vt / peak_int8, 4)}
            res[name]["variants"] = variants
    return res


def run_quantize(args, dev, stream, world, peaks, peak_src):
    """Quantisation prologue on one LLaMA-7B-layer activation (bf16
    [1, 32, 8192, 128], per-head scales): GB/s of the bf16 read + int8 write."""
    import torch

    import integer_only_quantized_b200 as ia
    shape = (1, 32, 8192, 128)
    n = 1
    for s_ in shape:
        n *= s_
    g = torch.Generator(device=dev)
    g.manual_seed(20251126)
    xs = [torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16) for _ in range(3)]
    out = torch.empty(shape, dtype=torch.int8, device=dev)
    scales = torch.empty(shape[1], dtype=torch.float32, device=dev)
    steps = max(10, min(args.steps, 60))
    torch.cuda.synchronize(dev)  # inputs made on the default stream are complete before `stream` reads them
    for i in range(max(3, args.warmup)):
        ia.quantize(xs[i % 3], True, out=out, scales=scales, stream=stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        ia.quantize(xs[i % 3], True, out=out, scales=scales, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    err = ia.device_error(stream)
    if err != ia.OK:
        raise RuntimeError(f"device error {err} ({ia.strerror(err)}) in the quantisation leg")
    algo = 3 * n  # 2 bytes read + 1 byte written per element
    gbs = algo / (ms * 1e-3) / 1e9
    return {"workload": "llama7b_layer_bf16_b1h32l8192d128", "value": round(aggregate_value(algo, world, ms * 1e-3) / 1e9, 1),
            "unit": "GB/s", "ms_per_call": round(ms, 5), "launches_per_call": 2, "bytes_per_call": algo,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": f"{peak_src} hbm_gbs",
                         "traffic": kernel_traffic("quant_fused_kernel", "llama7b_layer_bf16_b1h32l8192d128")},
            "l2": "inputs rotate over 3 copies (201 MB > 126 MB L2)"}


def run_forward_fp(args, dev, stream, world, peaks, peak_src):
    """The forward from bf16 activations (intattn_forward_fp) on the
    LLaMA-7B causal prefill shape: quantise q, k, v on the device, derive the
    head parameters on the device, integer forward; every launch of a call
    is inside the timed region."""
    import numpy as np
    import torch

    import integer_only_quantized_b200 as ia
    from integer_only_quantized_b200 import workloads as wl
    w = wl.WORKLOADS["llama7b_causal_l8192"]
    g = torch.Generator(device=dev)
    g.manual_seed(20251126)
    shape = (w.B, w.H, w.Lq, w.d)
    sets = [tuple(torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
                  for _ in range(3)) for _ in range(2)]  # two sets: 2 x 100.7 MB > L2
    out = torch.empty(shape, dtype=torch.int8, device=dev)
    ws = torch.empty(ia.forward_fp_workspace_size(w.B, w.H, w.Lq, w.Lk, w.d), dtype=torch.uint8, device=dev)
    s_o = np.full(w.H, 0.02, np.float32)
    call = lambda i: ia.forward_fp(*sets[i % 2], True, s_o, w.causal, w.clip_c, out=out, workspace=ws, stream=stream)
    steps = max(10, min(args.steps, 40))
    torch.cuda.synchronize(dev)  # inputs made on the default stream are complete before `stream` reads them
    for i in range(max(3, args.warmup)):
        call(i)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        call(i)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    err = ia.device_error(stream)
    if err != ia.OK:
        raise RuntimeError(f"device error {err} ({ia.strerror(err)}) in the forward from bf16")
    peak_int8, _ = _int8_peak(peaks, sustained=False)
    tops = w.effective_ops / (ms * 1e-3) / 1e12
    return {"workload": w.name + "_bf16_inputs", "value": round(aggregate_value(w.effective_ops, world, ms * 1e-3) / 1e12, 3),
            "unit": "TOPS", "ms_per_call": round(ms, 5), "launches_per_call": 8,
            "note": "bf16 q, k, v -> int8 out: three quantisations (2 launches each), device-side parameters, forward",
            "roofline": {"bound": "tensor", "achieved": round(tops, 3), "peak": round(peak_int8, 1), "unit": "TOPS",
                         "frac": round(tops / peak_int8, 4)},
            "l2": "inputs alternate between 2 sets (201 MB > 126 MB L2)"}


def run_zero_point(args, ia, dev, stream, world, peak_int8, base_ms):
    """The headline prefill with K and V as u8 codes carrying zero-points
    (the int8 codes re-expressed as code + 128 with zero-point 128, so the
    output bytes are the headline's): the cost of the zero-point path, timed
    exactly like the headline."""
    import dataclasses

    import numpy as np

    from integer_only_quantized_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    x = wl.make_inputs(w)
    xu = dataclasses.replace(x, k=(x.k.astype(np.int16) + 128).astype(np.uint8),
                             v=(x.v.astype(np.int16) + 128).astype(np.uint8))
    n = w.H if w.per_head else 1
    z = np.full(n, 128, np.int32)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head, z_k=z, z_v=z)
    nsets, _ = rotation(w)
    steps = max(10, min(args.steps, 40), nsets)
    ms, _ = time_prefill(ia, w, xu, dev, stream, steps, max(3, args.warmup), None, world, scales=sc)
    tops = w.effective_ops / (ms * 1e-3) / 1e12
    return {"workload": w.name + "_u8_kv_zero_points", "value": round(aggregate_value(w.effective_ops, world,
                                                                                      ms * 1e-3) / 1e12, 3),
            "unit": "TOPS", "ms_per_call": round(ms, 5), "launches_per_call": 1,
            "vs_symmetric": round(ms / base_ms, 4),
            "note": "u8 K and V with zero-point 128 per head: the MMA reads u8, and z_v sum P is subtracted "
                    "through one correction MMA per softmax team per query tile",
            "roofline": {"bound": "tensor", "achieved": round(tops, 3), "peak": round(peak_int8, 1), "unit": "TOPS",
                         "frac": round(tops / peak_int8, 4),
                         "traffic": kernel_traffic("prefill_kernel", w.name + "_u8_kv_zero_points")}}


def run_calibrate(args, dev, stream, world):
    """Adaptive clip thresholds (intattn_calibrate_clip) on the LLaMA-7B
    causal prefill codes: every 64th query row of each head sampled, the gap
    to its 32nd largest score.  Each sampled row's scores are computed once
    (dp4a, four rows of a head per CTA sharing the K reads) into shared
    memory, where three radix-select sweeps find the K-th largest: the
    counted work is sampled rows x valid keys x d multiply-adds.  Timed with
    CUDA events around whole calls (the call copies the gaps to the host and
    synchronises)."""
    import torch

    import integer_only_quantized_b200 as ia
    from integer_only_quantized_b200 import workloads as wl
    w = wl.WORKLOADS["llama7b_causal_l8192"]
    x = wl.make_inputs(w)
    q = torch.from_numpy(x.q).to(dev)
    k = torch.from_numpy(x.k).to(dev)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    keep, stride = 32, 64
    ws = torch.empty(max(ia.calibrate_workspace_size(w.B, w.H), 1), dtype=torch.uint8, device=dev)
    call = lambda: ia.calibrate_clip(q, k, sc, w.causal, keep, stride, workspace=ws, stream=stream)
    torch.cuda.synchronize(dev)  # inputs made on the default stream are complete before `stream` reads them
    for _ in range(max(3, args.warmup)):
        call()
    steps = max(5, min(args.steps, 20))
    barrier(world, dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        call()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    if ia.device_error(stream) != ia.OK:
        raise RuntimeError("a kernel wait timed out in calibrate_clip")
    rows = list(range(stride - 1, w.Lq, stride))
    off = w.Lk - w.Lq
    keys = sum(min(w.Lk, i + off + 1) if w.causal else w.Lk for i in rows) * w.B * w.H
    ops = keys * w.d * 2  # each sampled score once: int8 multiply-adds
    tops = ops / (ms * 1e-3) / 1e12
    # dp4a issues at half the FP32 rate: 64 per clock per SM, 8 int8 ops each
    peak = 148 * 64 * 8 * 1.965e9 / 1e12
    return {"workload": w.name + f"_keep{keep}_stride{stride}", "ms_per_call": round(ms, 5), "launches_per_call": 2,
            "sampled_rows": len(rows) * w.B * w.H, "scores_per_sweep": keys,
            "note": "memset of the gap buffer + gap kernel (scores in shared memory, radix select there); "
                    "thresholds from the gaps on the host",
            "value": round(aggregate_value(ops, world, ms * 1e-3) / 1e12, 3), "unit": "TOPS (dp4a int8)",
            "roofline": {"bound": "alu", "achieved": round(tops, 3), "peak": round(peak, 1), "unit": "TOPS",
                         "frac": round(tops / peak, 4), "peak_source": "148 SMs x 64 dp4a/clk x 8 ops x 1965 MHz",
                         "traffic": None}}


def run_gelu(args, dev, stream, world, peaks, peak_src):
    """Integer GELU over GPT-2-small MLP activations (int8 [16*1024, 3072]):
    GB/s of the int8 read + int8 write."""
    import torch

    import integer_only_quantized_b200 as ia
    from integer_only_quantized_b200 import workloads as wl
    name = "gpt2_small_mlp_gelu_b16_l1024_f3072"
    spec = wl.GELU_WORKLOADS[name]
    ins = [wl.gelu_inputs_torch(spec["tokens"], spec["features"], 20251126 + i, dev) for i in range(4)]
    xs = [c for c, _ in ins]
    s_x = ins[0][1]
    n = xs[0].numel()
    out = torch.empty_like(xs[0])
    steps = max(10, min(args.steps, 100))
    torch.cuda.synchronize(dev)  # inputs made on the default stream are complete before `stream` reads them
    for i in range(max(3, args.warmup)):
        ia.gelu(xs[i % 4], s_x, s_x, spec["c"], out=out, stream=stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        ia.gelu(xs[i % 4], s_x, s_x, spec["c"], out=out, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    algo = 2 * n  # 1 byte read + 1 byte written per element
    gbs = algo / (ms * 1e-3) / 1e9
    return {"workload": name, "value": round(aggregate_value(algo, world, ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "ms_per_call": round(ms, 5), "launches_per_call": 1, "bytes_per_call": algo,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": f"{peak_src} hbm_gbs",
                         "traffic": kernel_traffic("gelu_kernel", name)},
            "l2": "inputs rotate over 4 copies (201 MB > 126 MB L2)"}


def run_decode(args, dev, stream, world, peaks, peak_src, name):
    """Decode over the int8 (or packed int4) KV cache: GB/s of K/V cache rows
    + q + out."""
    import torch

    import integer_only_quantized_b200 as ia
    from integer_only_quantized_b200 import workloads as wl
    w = wl.WORKLOADS[name]
    x = wl.make_inputs_torch(w, dev)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    ws = torch.empty(ia.decode_workspace_size(w.B, w.H, w.Lk, w.d), dtype=torch.uint8, device=dev)
    out = torch.empty_like(x.q)
    if w.kv_bits == 4:
        kc, vc = wl.pack_int4_torch(x.k), wl.pack_int4_torch(x.v)
        del x.k, x.v
        call = lambda: ia.decode_int4(x.q, kc, vc, sc, w.Lk, w.clip_c, out=out, workspace=ws, stream=stream)
    else:
        call = lambda: ia.decode(x.q, x.k, x.v, sc, w.Lk, w.clip_c, out=out, workspace=ws, stream=stream)
    steps = max(10, min(args.steps, 100))
    torch.cuda.synchronize(dev)  # inputs made on the default stream are complete before `stream` reads them
    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        call()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    if ia.device_error(stream) != ia.OK:
        raise RuntimeError("a kernel wait timed out in decode")
    gbs = w.decode_bytes / (ms * 1e-3) / 1e9
    return {"workload": w.name, "value": round(aggregate_value(w.decode_bytes, world, ms * 1e-3) / 1e9, 1),
            "unit": "GB/s", "ms_per_call": round(ms, 5),
            # int4 rows of at most 4096 keys: Q.K^T and P.V (which also finds Z)
            "launches_per_call": 2 if (w.kv_bits == 4 and w.Lk <= 4096) else 3,
            "bytes_per_call": int(w.decode_bytes),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "peak_source": f"{peak_src} hbm_gbs",
                         "traffic": kernel_traffic("decode", w.name, "bytes_per_call"),
                         "traffic_unit": "DRAM bytes per call (all launches of one call)"},
            "kv_bits": w.kv_bits,
            "l2": f"K/V caches {2 * w.B * w.H * w.Lmax * w.d * w.kv_bits / 8 / 2**30:.0f} GiB > 126 MiB L2"}


# ------------------------------------------------------- CPU oracle legs
def _oracle_sample(w, x, seconds: float):
    """Time the oracle on whole (b, h) slices, in order and wrapping around,
    until about `seconds` of work (at least one slice)."""
    import oracle
    threads = os.cpu_count() or 1
    oracle.build()
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    done = 0
    t0 = time.perf_counter()
    while True:
        b, h = heads[done % len(heads)]
        sl = slice(h, h + 1)
        hsc = (lambda s: s[sl] if w.per_head else s)
        oracle.forward(x.q[b:b + 1, sl], x.k[b:b + 1, sl], x.v[b:b + 1, sl], w.per_head,
                       hsc(x.s_q), hsc(x.s_k), hsc(x.s_v), hsc(x.s_o), w.causal, w.clip_c,
                       nthreads=threads)
        done += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    ops = w.effective_ops / (w.B * w.H) * done
    return ops, dt, threads, (f"{done} (b, h) slices of {w.name} (all rows of each; "
                              f"{done / (w.B * w.H):.2f} passes over the workload)")


def cpu_baseline(w, x, seconds):
    ops, dt, threads, sample = _oracle_sample(w, x, seconds)
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": threads, "kind": "oracle",
            "sample": sample, "seconds": round(dt, 2)}


def run_reference(args):
    from integer_only_quantized_b200 import workloads as wl
    rank, _, world = dist_env()
    if rank != 0:
        return  # only rank 0 times the oracle; the other ranks do no work
    w = wl.WORKLOADS[args.workload]
    x = wl.make_inputs(w)
    per_step = max(0.5, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        _oracle_sample(w, x, per_step)
    total_ops, total_t = 0.0, 0.0
    sample = threads = None
    for _ in range(args.steps):
        ops, dt, threads, sample = _oracle_sample(w, x, per_step)
        total_ops += ops
        total_t += dt
    value = total_ops / total_t / 1e12
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": threads,
                             "kind": "oracle", "sample": f"each step: {sample}"},
            "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    elif args.leg:
        run_leg(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
