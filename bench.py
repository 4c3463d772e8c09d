#!/usr/bin/env python
"""Benchmark of the sparse MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one moe_forward call (router, dispatch, routed experts, shared
expert, combine) over one batch of T synthetic tokens already resident in
HBM.  With N > 1 (torchrun, one process per GPU) every rank runs its own
batch of T tokens against replicated weights: the layer has no data-path
exchange, so there is no collective besides the timing reduction (weak
scaling).  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (fp64 NumPy) on the host cores on
bounded samples of the same workload; it is the slow reference arm.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import moe_synth as ms  # noqa: E402

METRIC = "MoE-layer fwd tokens/s at 1 B200; % of bf16 tensor peak or HBM roofline"
DEFAULT_CONFIG = "glm5_skewed_prefill_bf16"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Files whose content defines the GEMM kernel measured by the recorded ncu
# counters (a change voids the recorded traffic figure).
GEMM_SOURCES = ["sparse_mixture_experts_logits_b200/csrc/gemm_swap_sm100.cuh",
                "sparse_mixture_experts_logits_b200/csrc/gemm_swap_sm100.cu",
                "sparse_mixture_experts_logits_b200/csrc/common.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU-baseline run time")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="target run time of the whole --impl reference run")
    ap.add_argument("--T", type=int, default=None, help="override tokens per GPU (profiling runs)")
    ap.add_argument("--M", type=int, default=None, help="override routed experts (profiling runs)")
    ap.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward"],
                    help="backward: time moe_backward (all gradients of the layer) instead of the forward")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: each of the N ranks owns M/N experts, rows exchanged by all-to-all")
    ap.add_argument("--capacity-factor", type=float, default=2.0,
                    help="--ep: each expert takes at most ceil(f T k / M) rows from each rank (fixed splits)")
    return ap.parse_args()


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def dist_init(world, local_rank, backend="nccl"):
    if world <= 1:
        return None
    import torch.distributed as dist
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    else:
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return dist


def token_rows(rank: int, T: int) -> tuple[int, int]:
    """Rows of the global synthetic token stream that rank `rank` processes."""
    return rank * T, (rank + 1) * T


def max_over_ranks(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------
# measurement helpers
# --------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def e2e_overlapped(K, dev, stream, stage_in, compute, stage_out, flush, dist):
    """Device ms per step of K end-to-end steps, each with its own host->device
    copy of the inputs (pinned host memory), the layer, and a device->host copy
    of its result.  Two buffer sets alternate: step i's input copy (copy stream
    one) and step i-1's result copy (copy stream two) run on the copy engines
    while step i-1 / i computes, as a caller streaming batches through the
    layer would run them.  Timed from the first copy's start to the last
    copy's end (events on the copy streams), divided by K, max over ranks.
    stage_in(b, s), compute(b, s), stage_out(b, s) enqueue buffer set b's
    work on stream s."""
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n, start=None, end=None):
        for b in range(2):  # nothing pending on either buffer set
            ev_comp[b].record(stream)
            ev_out[b].record(s_out)
        if start is not None:
            s_in.wait_event(ev_comp[1])
            start.record(s_in)
        for i in range(n):
            b = i & 1
            s_in.wait_event(ev_comp[b])           # step i-2 has read its inputs
            stage_in(b, s_in)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])          # step i-2's result has left
            flush.zero_()
            compute(b, stream)
            ev_comp[b].record(stream)
            s_out.wait_event(ev_comp[b])
            stage_out(b, s_out)
            ev_out[b].record(s_out)
        if end is not None:
            end.record(s_out)

    run(4)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(K, t0, t1)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return max_over_ranks(dist, t0.elapsed_time(t1) / K, dev)


E2E_NOTE = ("each step copies its own inputs in from pinned host memory and its result out; two buffer sets "
            "alternate so that the copies run on the copy engines under the neighbouring steps' compute")


def wait_on_last(events):
    """Blocks until the last of `events` completes by polling it with short
    sleeps: the host thread holds no lock while it waits, so the clock
    sampler keeps reading NVML through the timed region."""
    while events and not events[-1].query():
        time.sleep(0.0005)


class ClockSampler:
    """SM clocks, power and clock-event reasons sampled DURING the timed region.

    NVML is read from a background thread every few milliseconds between
    start() and stop(), so even a timed region of a few tens of milliseconds
    (decode) gets samples; without NVML, nvidia-smi's own -lms loop is the
    fallback.  Only reads: no clock or other setting is touched."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.rows = []
        self.stopping = False
        self.nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = None
            try:  # the CUDA device's own NVML handle, whatever CUDA_VISIBLE_DEVICES says
                props = torch.cuda.get_device_properties(gpu_index)
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.nvml = (pynvml, handle)
        except Exception:
            self.nvml = None

    def _poll(self):
        pynvml, h = self.nvml
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stopping:
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                reasons = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                power = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.rows.append((float(sm), float(smax), power, int(reasons)))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.nvml is not None:
            import threading
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stopping = True
            self.thread.join(timeout=5)
            rows = self.rows
            if not rows:
                return None
            reasons = sorted(n for n, bit in self.REASONS.items() if any(r[3] & bit for r in rows))
            return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                    "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows),
                    "source": "nvml, every 5 ms during the timed region"}
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None, "source": "nvidia-smi -lms 200"}


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_stage: str, workload: str, units_scale: float = 1.0):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when absent or taken on a different kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    e = rec.get(workload, {}).get(kernel_stage)
    if not e or e.get("source_hash") != source_hash(GEMM_SOURCES):
        return None
    return e["dram_bytes_per_launch"] * units_scale


def stage_work(cfg, counts):
    """Algorithmic FLOPs and bytes of each stage (active experts only;
    intermediates and padding rows are not credited)."""
    T, D, M, k, I = cfg["T"], cfg["D"], cfg["M"], cfg["k"], cfg["I"]
    es = 2 if cfg["dtype"] == "bf16" else 4
    swiglu = cfg["act"] == "swiglu"
    n1 = 2 * I if swiglu else I
    touched = int((counts > 0).sum())
    pairs = T * k
    bias = (not swiglu) and cfg.get("has_bias")
    Ish = cfg.get("I_sh") or 0
    w = {
        "route": (2.0 * T * D * M, (T * D + D * M) * es + T * k * 8),
        "dispatch": (0.0, T * k * 4 * 5),
        "gather": (0.0, 2.0 * pairs * D * es),
        "expert_up": (2.0 * pairs * D * n1, touched * (n1 * D + (I if bias else 0)) * es),
        "expert_down": (2.0 * pairs * I * D, touched * (D * I + (D if bias else 0)) * es),
        "shared_up": (2.0 * T * D * 2 * Ish, 2.0 * Ish * D * es),
        "shared_down": (2.0 * T * Ish * D, D * Ish * es),
        "combine": (0.0, T * D * es),
    }
    return w


def workload_config(args):
    over = {}
    if args.T is not None:
        over["T"] = args.T
    if args.M is not None:
        over["M"] = args.M
    return ms.get_config(args.config, **over)


def is_dense(cfg) -> bool:
    return cfg["name"] in ms.DENSE_CONFIGS


def metric_name(cfg) -> str:
    return METRIC.replace("MoE-layer", "dense FFN layer") if is_dense(cfg) else METRIC


# --------------------------------------------------------------------------
# the GPU arm
# --------------------------------------------------------------------------

def run_ours(args):
    import sparse_mixture_experts_logits_b200 as B

    rank, local_rank, world = dist_env()
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = dist_init(world, local_rank)

    cfg = workload_config(args)
    T, D = cfg["T"], cfg["D"]
    inp = ms.layer_inputs(dict(cfg, T=1), dev)  # weights; x below
    r0, r1 = token_rows(rank, T)
    x = ms.normal_rows(torch.arange(r0, r1, device=dev), D, 1.0, ms._key(cfg, "x"),
                       ms.act_dtype(cfg))
    inp["x"] = x
    layer = B.MoELayer(cfg, inp)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fwd():
        B.moe_forward(layer.desc, layer.weights, x.data_ptr(), y.data_ptr(), layer.ws_ptr,
                      layer.ws_bytes, sh)

    for _ in range(max(3, args.warmup)):
        fwd()
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise RuntimeError("device status flag set during warm-up")
    counts = layer.view("counts").cpu().numpy()

    K = args.steps
    n_ev = B.NUM_STAGE_EVENTS
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(K)]
    for evs in [starts, ends] + stage_ev:  # torch creates the CUDA event on first record
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for i in range(K):
        flush.zero_()  # L2 flush between steps, outside the timed events
        starts[i].record(stream)
        B.moe_forward_profiled(layer.desc, layer.weights, x.data_ptr(), y.data_ptr(), layer.ws_ptr,
                               layer.ws_bytes, sh, [e.cuda_event for e in stage_ev[i]])
        ends[i].record(stream)
    wait_on_last(ends)  # sleeps, so that the clock sampler thread gets the GIL
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if dist is not None:
        dist.barrier()
    step_ms = [starts[i].elapsed_time(ends[i]) for i in range(K)]
    ms_local = sum(step_ms) / K
    stage_ms = {}
    for s, name in enumerate(B.STAGE_NAMES):
        stage_ms[name] = sum(stage_ev[i][s].elapsed_time(stage_ev[i][s + 1]) for i in range(K)) / K
    ms_step = max_over_ranks(dist, ms_local, dev)
    if layer.device_status() != 0:
        raise RuntimeError("device status flag set during the timed steps")

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        x_host = x.cpu().pin_memory()
        y_host = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(x) for _ in range(2)]
        y_dev = [torch.empty_like(y) for _ in range(2)]
        # the layer's workspace is shared by the two buffer sets: the steps run in order on `stream`

        def stage_in(b, s):
            with torch.cuda.stream(s):
                x_dev[b].copy_(x_host, non_blocking=True)

        def compute(b, s):
            B.moe_forward(layer.desc, layer.weights, x_dev[b].data_ptr(), y_dev[b].data_ptr(), layer.ws_ptr,
                          layer.ws_bytes, s.cuda_stream)

        def stage_out(b, s):
            with torch.cuda.stream(s):
                y_host[b].copy_(y_dev[b], non_blocking=True)

        e2e_ms = e2e_overlapped(K, dev, stream, stage_in, compute, stage_out, flush, dist)
        if not torch.equal(y_host[(K - 1) & 1], y.cpu()):
            raise RuntimeError("the end-to-end steps' result differs from the timed steps'")
        nbytes = x.numel() * x.element_size()
        e2e = {"value": world * T / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes, "note": E2E_NOTE}

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    peaks, peak_src = load_peaks()
    work = stage_work(cfg, counts)
    flops_total, bytes_total = B.moe_algorithmic_work(layer.desc, counts)
    gemm_stages = [s for s in ("expert_up", "expert_down", "shared_up", "shared_down") if stage_ms[s] > 0.002]
    dom = max(gemm_stages, key=lambda s: stage_ms[s])
    f, b = work[dom]
    t_s = stage_ms[dom] / 1e3
    # The timed region is a short run of steps (tens of ms, not a seconds-long
    # loop at the power cap), so the burst tensor figure is the denominator;
    # the fraction of the sustained figure is reported beside it.
    peak_tf = peaks["bf16_tflops"]
    peak_tf_sust = peaks.get("bf16_tflops_sustained", peak_tf)
    peak_bw = peaks["hbm_gbs"]
    t_f, t_b = f / (peak_tf * 1e12), b / (peak_bw * 1e9)
    if t_f >= t_b:
        roof = {"bound": "tensor", "achieved": f / t_s / 1e12, "peak": peak_tf, "unit": "TFLOP/s"}
        roof["frac_of_sustained_peak"] = roof["achieved"] / peak_tf_sust
    else:
        roof = {"bound": "hbm", "achieved": b / t_s / 1e9, "peak": peak_bw, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(dom, args.config)
    few_rows = cfg["T"] * cfg["k"] < 4 * cfg["M"]  # the library's decode-shape choice of expert GEMM
    routed_kernel = "moe_gemm_sm100_kernel<EPI, 1>" if few_rows else "moe_gemm_swap_kernel"
    roof["kernel"] = f"{routed_kernel if dom.startswith('expert') else 'moe_gemm_swap_kernel'} ({dom})"
    roof["peak_source"] = (f"{peak_src}: " + ("bf16_tflops (burst; the timed region is ms long)"
                                             if roof["bound"] == "tensor" else "hbm_gbs"))
    roof["algorithmic"] = {"flops": f, "bytes": b}
    t_layer_ideal = max(flops_total / (peak_tf * 1e12), bytes_total / (peak_bw * 1e9))
    t_layer_ideal_sust = max(flops_total / (peak_tf_sust * 1e12), bytes_total / (peak_bw * 1e9))

    out = {
        "metric": METRIC,
        "value": world * T / (ms_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg["dtype"],
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": {"workload": args.config + ("" if cfg["named"] else " (overridden: T=%d, M=%d)" % (T, cfg["M"])),
                   "T_per_gpu": T, "D": D, "M": cfg["M"], "k": cfg["k"],
                   "I": cfg["I"], "I_sh": cfg.get("I_sh", 0), "gate": cfg["gate"], "act": cfg["act"],
                   "l2": "flushed between steps (256 MiB write outside the timed events)",
                   "parallelism": f"replicas x{world} (token batches, no data-path collective)"},
        "roofline": roof,
        "layer": {"tflops": flops_total / (ms_step / 1e3) / 1e12,
                  "algorithmic_flops": flops_total, "algorithmic_bytes": bytes_total,
                  "ideal_ms": t_layer_ideal * 1e3, "frac_of_ideal": t_layer_ideal / (ms_step / 1e3),
                  "frac_of_ideal_sustained": t_layer_ideal_sust / (ms_step / 1e3)},
        "stages_ms": stage_ms,
        "e2e": e2e,
        "gpu_launches": B.moe_forward_launch_count(layer.desc) * K,
        "clocks": clocks,
        "routing": {"touched_experts": int((counts > 0).sum()), "max_over_mean":
                    float(counts.max() / max(1e-9, counts.mean())),
                    "min": int(counts.min()), "median": float(np.median(counts)), "max": int(counts.max()),
                    "cv": float(counts.std() / max(1e-9, counts.mean()))},
        "reporting": glam_reporting(cfg, stage_ms, ms_step),
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, inp, args.cpu_seconds)
    print(json.dumps(out), flush=True)
    del layer
    if dist is not None:
        dist.destroy_process_group()


def glam_reporting(cfg, stage_ms, ms_step):
    """The quantities the GLaM note's "Capacity, Active Compute, and
    Reporting" table keeps apart: total parameters, active parameters per
    token, FLOPs per token, routing overhead (gate, dispatch, expert batching,
    combination) and the wall-clock cost."""
    D, M, k, I, Ish = cfg["D"], cfg["M"], cfg["k"], cfg["I"], cfg.get("I_sh") or 0
    swiglu = cfg["act"] == "swiglu"
    expert = (3 if swiglu else 2) * D * I + ((I + D) if cfg.get("has_bias") and not swiglu else 0)
    shared = 3 * D * Ish
    router = D * M + (M if cfg.get("e_bias") is not None else 0)
    active = router + k * expert + shared
    matmul_active = D * M + k * (3 if swiglu else 2) * D * I + shared
    overhead = {n: stage_ms.get(n, 0.0) for n in ("route", "dispatch", "gather", "combine")}
    return {"total_params": router + M * expert + shared, "active_params_per_token": active,
            "flops_per_token": 2 * matmul_active,
            "routing_overhead_ms": overhead, "routing_overhead_share": sum(overhead.values()) / ms_step,
            "wall_clock_ms": ms_step}


def dense_stage_work(cfg):
    """Algorithmic FLOPs and bytes of the dense layer's two GEMMs (weights,
    biases and the addend; the hidden activations are not credited)."""
    T, D, I = cfg["T"], cfg["D"], cfg["I"]
    es = 2 if cfg["dtype"] == "bf16" else 4
    n1 = 2 * I if cfg["act"] == "swiglu" else I
    bias = cfg["act"] != "swiglu" and cfg.get("has_bias")
    return {
        "dense_up": (2.0 * T * D * n1, (n1 * D + (I if bias else 0) + T * D) * es),
        "dense_down": (2.0 * T * I * D, (D * I + (D if bias else 0) + 2 * T * D) * es),
    }


def library_dense_ms(cfg, inp, flush, stream, steps=5):
    """The same dense layer through PyTorch's library GEMMs (cuBLAS), timed
    the same way: context for the tensor-core kernels, not the product."""
    import torch.nn.functional as F
    x, a = inp["x"], inp["addend"]
    I = cfg["I"]

    def layer():
        if cfg["act"] == "swiglu":
            gu = F.linear(x, inp["w1"])
            h = F.silu(gu[:, :I]) * gu[:, I:]
            return a + F.linear(h, inp["w2"])
        h = F.gelu(F.linear(x, inp["w1"], inp.get("b1")), approximate="tanh")
        return a + F.linear(h, inp["w2"], inp.get("b2"))

    for _ in range(3):
        layer()
    times = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return sum(times) / len(times)


def run_dense(args):
    """The dense FFN layer of the GLaM note's interleaved blocks:
    y = addend + FFN(x), through moe_dense_ffn_profiled."""
    import sparse_mixture_experts_logits_b200 as B

    rank, local_rank, world = dist_env()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = dist_init(world, local_rank)
    cfg = workload_config(args)
    T, D = cfg["T"], cfg["D"]
    inp = ms.dense_inputs(dict(cfg, T=1), dev)
    r0, r1 = token_rows(rank, T)
    rows = torch.arange(r0, r1, device=dev)
    inp["x"] = ms.normal_rows(rows, D, 1.0, ms._key(cfg, "x"), ms.act_dtype(cfg))
    inp["addend"] = ms.normal_rows(rows, D, 1.0, ms._key(cfg, "addend"), ms.act_dtype(cfg))
    layer = B.DenseLayer(cfg, inp)
    x, a = inp["x"], inp["addend"]
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    wargs = layer.args()

    for _ in range(max(3, args.warmup)):
        B.moe_dense_ffn(layer.desc, *wargs, x.data_ptr(), a.data_ptr(), y.data_ptr(), layer.ws_ptr,
                        layer.ws_bytes, sh)
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise RuntimeError("device status flag set during warm-up")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(B.NUM_DENSE_EVENTS)] for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for evs in ev + [ends]:
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for i in range(K):
        flush.zero_()
        B.moe_dense_ffn_profiled(layer.desc, *wargs, x.data_ptr(), a.data_ptr(), y.data_ptr(), layer.ws_ptr,
                                 layer.ws_bytes, sh, [e.cuda_event for e in ev[i]])
        ends[i].record(stream)
    wait_on_last(ends)  # sleeps, so that the clock sampler thread gets the GIL
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if dist is not None:
        dist.barrier()
    if layer.device_status() != 0:
        raise RuntimeError("device status flag set during the timed steps")
    ms_local = sum(ev[i][0].elapsed_time(ends[i]) for i in range(K)) / K
    stage_ms = {"dense_up": sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)) / K,
                "dense_down": sum(ev[i][1].elapsed_time(ev[i][2]) for i in range(K)) / K}
    ms_step = max_over_ranks(dist, ms_local, dev)

    e2e = None
    if not args.no_e2e:
        x_host = x.cpu().pin_memory()
        a_host = a.cpu().pin_memory()
        y_host = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(x) for _ in range(2)]
        a_dev = [torch.empty_like(a) for _ in range(2)]
        y_dev = [torch.empty_like(y) for _ in range(2)]

        def stage_in(b, s):
            with torch.cuda.stream(s):
                x_dev[b].copy_(x_host, non_blocking=True)
                a_dev[b].copy_(a_host, non_blocking=True)

        def compute(b, s):
            B.moe_dense_ffn(layer.desc, *wargs, x_dev[b].data_ptr(), a_dev[b].data_ptr(), y_dev[b].data_ptr(),
                            layer.ws_ptr, layer.ws_bytes, s.cuda_stream)

        def stage_out(b, s):
            with torch.cuda.stream(s):
                y_host[b].copy_(y_dev[b], non_blocking=True)

        e2e_ms = e2e_overlapped(K, dev, stream, stage_in, compute, stage_out, flush, dist)
        if not torch.equal(y_host[(K - 1) & 1], y.cpu()):
            raise RuntimeError("the end-to-end steps' result differs from the timed steps'")
        nbytes = x.numel() * x.element_size()
        e2e = {"value": world * T / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 2 * nbytes, "d2h_bytes_per_step": nbytes, "note": E2E_NOTE}

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    lib_ms = library_dense_ms(cfg, inp, flush, stream) if world == 1 else None
    peaks, peak_src = load_peaks()
    work = dense_stage_work(cfg)
    dom = max(stage_ms, key=lambda k: stage_ms[k])
    f, b = work[dom]
    t_s = stage_ms[dom] / 1e3
    peak_tf = peaks["bf16_tflops"]  # burst: the timed region is ms long
    peak_bw = peaks["hbm_gbs"]
    if f / (peak_tf * 1e12) >= b / (peak_bw * 1e9):
        roof = {"bound": "tensor", "achieved": f / t_s / 1e12, "peak": peak_tf, "unit": "TFLOP/s",
                "frac_of_sustained_peak": f / t_s / 1e12 / peaks.get("bf16_tflops_sustained", peak_tf)}
    else:
        roof = {"bound": "hbm", "achieved": b / t_s / 1e9, "peak": peak_bw, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(dom, args.config)
    roof["kernel"] = f"moe_gemm_swap_kernel ({dom})"
    roof["peak_source"] = (f"{peak_src}: " + ("bf16_tflops (burst; the timed region is ms long)"
                                             if roof["bound"] == "tensor" else "hbm_gbs"))
    roof["algorithmic"] = {"flops": f, "bytes": b}
    flops_total = sum(v[0] for v in work.values())
    out = {
        "metric": metric_name(cfg),
        "value": world * T / (ms_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg["dtype"],
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": {"workload": args.config + ("" if cfg["T"] == ms.DENSE_CONFIGS[cfg["name"]]["T"]
                                              else " (overridden: T=%d)" % T),
                   "T_per_gpu": T, "D": D, "I": cfg["I"], "act": cfg["act"],
                   "has_bias": int(bool(cfg.get("has_bias"))), "addend": True,
                   "l2": "flushed between steps (256 MiB write outside the timed events)",
                   "parallelism": f"replicas x{world} (token batches, no data-path collective)"},
        "roofline": roof,
        "layer": {"tflops": flops_total / (ms_step / 1e3) / 1e12, "algorithmic_flops": flops_total},
        "stages_ms": stage_ms,
        "library_gemms": None if lib_ms is None else {
            "what": "the same layer through torch.nn.functional.linear (cuBLAS) and torch activations",
            "ms_per_step": lib_ms, "tflops": flops_total / (lib_ms / 1e3) / 1e12},
        "e2e": e2e,
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, inp, args.cpu_seconds)
    print(json.dumps(out), flush=True)
    del layer
    if dist is not None:
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# the oracle on the host cores
# --------------------------------------------------------------------------

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(max(i.get("num_threads", 1) for i in info)), info[0].get("internal_api", "blas")
    except Exception:
        pass
    return os.cpu_count() or 1, "unknown"


class OracleRunner:
    """Runs the CPU oracle on token blocks of one workload.  Weights live on
    the host as bf16 and are widened to fp64 per expert when used, as the
    oracle does at full size."""

    def __init__(self, cfg, inp):
        import oracle
        self.oracle = oracle
        self.cfg = cfg
        self.x = inp["x"]
        host = {k: (None if v is None else v.cpu()) for k, v in inp.items() if k != "x"}
        self.w_r = host["w_r"].double().numpy()
        self.e_bias = None if host["e_bias"] is None else host["e_bias"].double().numpy()
        self.host = host
        self.shared = None
        if cfg.get("I_sh"):
            self.shared = (host["sh_w1"].double().numpy(), host["sh_w2"].double().numpy())

    def get_expert(self, e):
        h = self.host
        return (h["w1"][e].double().numpy(), h["w2"][e].double().numpy(),
                None if h["b1"] is None else h["b1"][e].double().numpy(),
                None if h["b2"] is None else h["b2"][e].double().numpy())

    def x_block(self, t0, n):
        T = self.x.shape[0]
        rows = torch.arange(t0, t0 + n) % T
        return self.x[rows.to(self.x.device)].double().cpu().numpy()

    def run(self, xs):
        c = self.cfg
        r = self.oracle.route(xs, self.w_r, self.e_bias, c["k"], c["gate"], c["norm_topk_prob"],
                              c["alpha"], c["eps"], c.get("n_group", 1) or 1, c.get("topk_group", 1) or 1)
        return self.oracle.moe_tokens(xs, r["idx"], r["w"], c["act"], self.get_expert, self.shared)


class DenseOracleRunner:
    """The CPU oracle's dense FFN layer (with its addend) on token blocks."""

    def __init__(self, cfg, inp):
        import oracle
        self.oracle = oracle
        self.cfg = cfg
        self.x = inp["x"]
        self.addend = inp["addend"]
        host = {k: (None if v is None else v.cpu().double().numpy()) for k, v in inp.items()
                if k not in ("x", "addend")}
        self.w = host

    def x_block(self, t0, n):
        T = self.x.shape[0]
        rows = (torch.arange(t0, t0 + n) % T).to(self.x.device)
        return self.x[rows].double().cpu().numpy(), self.addend[rows].double().cpu().numpy()

    def run(self, block):
        xs, a = block
        w = self.w
        return self.oracle.dense_layer(xs, self.cfg["act"], w["w1"], w["w2"], w.get("b1"), w.get("b2"),
                                       addend=a)


def cpu_baseline(cfg, inp, target_s):
    runner = DenseOracleRunner(cfg, inp) if is_dense(cfg) else OracleRunner(cfg, inp)
    n = 16
    while True:
        xs = runner.x_block(0, n)
        t0 = time.perf_counter()
        runner.run(xs)
        dt = time.perf_counter() - t0
        if dt >= target_s * 0.5 or n >= cfg["T"]:
            break
        n = int(min(cfg["T"], max(2 * n, n * target_s / max(dt, 1e-3))))
    cores, api = _blas_threads()
    widen = ("weights widened from bf16 once, outside the timed run" if is_dense(cfg) else
             "weights widened from bf16 per expert inside the timed run")
    return {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} of the workload's {cfg['T']} tokens through the fp64 NumPy oracle "
                      f"({api} BLAS); {widen}",
            "seconds": dt}


def run_reference(args):
    rank, local_rank, world = dist_env()
    if rank != 0:
        return
    cfg = workload_config(args)
    dev = torch.device("cuda", local_rank) if torch.cuda.is_available() else torch.device("cpu")
    if is_dense(cfg):
        runner = DenseOracleRunner(cfg, ms.dense_inputs(cfg, dev))
    else:
        runner = OracleRunner(cfg, ms.layer_inputs(cfg, dev))
    # size one step's token sample from a probe so that the whole run stays short
    probe_n = 8
    t0 = time.perf_counter()
    runner.run(runner.x_block(0, probe_n))
    per_step_budget = max(0.05, args.ref_seconds / max(1, args.steps + args.warmup))
    dt = time.perf_counter() - t0
    n = int(max(4, min(cfg["T"], probe_n * per_step_budget / max(dt, 1e-3))))
    cursor = 0
    for _ in range(args.warmup):
        runner.run(runner.x_block(cursor, n))
        cursor += n
    times = []
    for _ in range(args.steps):
        xs = runner.x_block(cursor, n)
        cursor += n
        t0 = time.perf_counter()
        runner.run(xs)
        times.append(time.perf_counter() - t0)
    mean_s = sum(times) / len(times)
    value = n / mean_s
    cores, api = _blas_threads()
    sample = (f"{n} consecutive tokens per step of the {cfg['T']}-token workload, fp64 NumPy oracle "
              f"({api} BLAS); every step widens the bf16 weights of each expert its tokens chose to fp64, "
              f"which dominates at this sample size (the GPU line's cpu_baseline runs one large block "
              f"instead, so each expert is widened once for many tokens)")
    out = {
        "impl": "reference", "metric": metric_name(cfg), "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": ({"workload": args.config, "T_per_gpu": cfg["T"], "D": cfg["D"], "I": cfg["I"],
                    "act": cfg["act"]} if is_dense(cfg) else
                   {"workload": args.config, "T_per_gpu": cfg["T"], "D": cfg["D"], "M": cfg["M"],
                    "k": cfg["k"], "I": cfg["I"], "I_sh": cfg.get("I_sh", 0)}),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def backward_cpu_baseline(cfg, inp, dy, idx, target_s, max_experts=16):
    """The fp64 backward oracle on the first tokens of the workload, each
    with only the experts it chose (its gradients do not depend on the
    others); the sample grows while its experts fit in host memory."""
    import oracle

    f64 = lambda t: t.detach().to(torch.float64).cpu().numpy()  # noqa: E731
    n = 1
    while True:
        used = np.unique(idx[:n])
        pos = {int(e): i for i, e in enumerate(used)}
        sel = torch.as_tensor(used.astype(np.int64), device=inp["w1"].device)
        sub = {"x": f64(inp["x"][:n]), "w_r": f64(inp["w_r"][:, sel])}
        for k in ("e_bias", "w1", "w2", "b1", "b2"):
            sub[k] = None if inp.get(k) is None else f64(inp[k][sel])
        for k in ("sh_w1", "sh_w2"):
            sub[k] = None if inp.get(k) is None else f64(inp[k])
        sub_idx = np.vectorize(lambda e: pos[int(e)])(idx[:n])
        sub_cfg = dict(cfg, T=n, M=len(used), n_group=1, topk_group=1)
        dyh = f64(dy[:n])
        t0 = time.perf_counter()
        oracle.moe_backward.moe_backward(sub_cfg, sub, dyh, idx=sub_idx)
        dt = time.perf_counter() - t0
        n2 = min(cfg["T"], 2 * n)
        if dt >= target_s * 0.3 or n2 == n or len(np.unique(idx[:n2])) > max_experts:
            break
        n = n2
    cores, api = _blas_threads()
    return {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} tokens of the workload with the {len(used)} experts they chose, fp64 NumPy "
                      f"backward oracle ({api} BLAS); weights widened outside the timed run",
            "seconds": dt}


def run_backward(args):
    """One step = moe_backward over the workload's tokens: the routing and
    the experts' forward values recomputed, then every gradient of the layer."""
    import sparse_mixture_experts_logits_b200 as B

    rank, local_rank, world = dist_env()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = dist_init(world, local_rank)
    cfg = workload_config(args)
    T, D = cfg["T"], cfg["D"]
    inp = ms.layer_inputs(dict(cfg, T=1), dev)
    r0, r1 = token_rows(rank, T)
    rows = torch.arange(r0, r1, device=dev)
    inp["x"] = ms.normal_rows(rows, D, 1.0, ms._key(cfg, "x"), ms.act_dtype(cfg))
    dy = ms.normal_rows(rows, D, 1.0, ms._key(cfg, "dy"), ms.act_dtype(cfg))
    layer = B.MoELayer(cfg, inp)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    grads = layer.backward(inp["x"], dy)
    for _ in range(max(3, args.warmup) - 1):
        layer.backward(inp["x"], dy, grads=grads)
    torch.cuda.synchronize()
    if layer.backward_status() != 0:
        raise RuntimeError("device status flag set during warm-up")
    counts = layer.backward_view("counts").cpu().numpy()
    idx = layer.backward_view("topk_idx").cpu().numpy()
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for i in range(K):
        flush.zero_()
        starts[i].record(stream)
        layer.backward(inp["x"], dy, grads=grads)
        ends[i].record(stream)
    wait_on_last(ends)  # sleeps, so that the clock sampler thread gets the GIL
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if dist is not None:
        dist.barrier()
    ms_step = max_over_ranks(dist, sum(starts[i].elapsed_time(ends[i]) for i in range(K)) / K, dev)
    if layer.backward_status() != 0:
        raise RuntimeError("device status flag set during the timed steps")
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    peaks, peak_src = load_peaks()
    fwd_flops, _ = B.moe_algorithmic_work(layer.desc, counts)
    # every GEMM of the layer has two in the backward (input and weight gradient)
    flops = 2.0 * fwd_flops
    peak_tf = peaks["bf16_tflops"]
    achieved = flops / (ms_step / 1e3) / 1e12
    # the CUDA-core fp32 FMA rate: 148 SMs x 128 lanes x 2 FLOP at the 1965 MHz clock ceiling
    simt_peak = 148 * 128 * 2 * 1.965e9 / 1e12
    tc = cfg["dtype"] == "bf16"
    out = {
        "metric": "MoE layer backward throughput (all gradients; routing and expert forward recomputed)",
        "value": world * T / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if tc else "f32",
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": {"workload": args.config, "T_per_gpu": T, "D": D, "M": cfg["M"], "k": cfg["k"],
                   "I": cfg["I"], "I_sh": cfg.get("I_sh", 0), "inputs": cfg["dtype"],
                   "arithmetic": ("bf16 operands on tcgen05, fp32 accumulation (moe_gemm_swap_kernel: forward, "
                                  "input-gradient and grouped-K weight-gradient layouts)") if tc else
                   "fp32 on the CUDA cores",
                   "l2": "flushed between steps (256 MiB write outside the timed events)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved / peak_tf, "traffic": None,
                     "kernel": ("the whole step (moe_gemm_swap_kernel launches hold most of it; see the launch list)"
                                if tc else "the whole step (bwd_gemm_kernel launches hold most of it)"),
                     "peak_source": f"{peak_src}: bf16_tflops (burst)",
                     "algorithmic": {"flops": flops, "note": "2 x forward FLOPs; the recompute is not counted"},
                     "frac_of_fp32_simt_peak": achieved / simt_peak},
        "e2e": None,
        "gpu_launches": B.moe_backward_launch_count(layer.desc) * K,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = backward_cpu_baseline(cfg, inp, dy, idx, args.cpu_seconds)
    print(json.dumps(out), flush=True)
    del layer
    if dist is not None:
        dist.destroy_process_group()


def run_ep(args):
    """One step = the expert-parallel forward (sparse_mixture_experts_logits_b200.ep) on
    every rank's own T tokens: route, exchange, local experts, exchange back, combine."""
    import sparse_mixture_experts_logits_b200 as B
    from sparse_mixture_experts_logits_b200 import ep

    rank, local_rank, world = dist_env()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = dist_init(world, local_rank)
    cfg = workload_config(args)
    T, D = cfg["T"], cfg["D"]
    full = ms.layer_inputs(dict(cfg, T=1), dev)
    mine = ep.local_expert_tensors(full, rank, world)
    del full
    r0, r1 = token_rows(rank, T)
    x = ms.normal_rows(torch.arange(r0, r1, device=dev), D, 1.0, ms._key(cfg, "x"), ms.act_dtype(cfg))
    layer = ep.ExpertParallelMoE(cfg, mine, rank, world, capacity_factor=args.capacity_factor)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        layer.forward(x)
    torch.cuda.synchronize()
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for i in range(K):
        flush.zero_()
        starts[i].record(stream)
        layer.forward(x)
        ends[i].record(stream)
    wait_on_last(ends)  # sleeps, so that the clock sampler thread gets the GIL
    torch.cuda.synchronize()
    launches = K * layer.launch_count(T)
    bufs = layer.buffers(T, x.dtype)
    kept_sent = int(bufs["kept"].sum().item())          # after the timed steps: the same every step
    kept_recv = int(bufs["recv_kept"].sum().item())
    clocks = sampler.stop() if sampler else None
    if dist is not None:
        dist.barrier()
    ms_step = max_over_ranks(dist, sum(starts[i].elapsed_time(ends[i]) for i in range(K)) / K, dev)
    if any(layer.status.tolist()):
        raise RuntimeError("device status flag set during the timed steps")
    if rank == 0:
        out = {
            "metric": "MoE layer forward throughput, expert-parallel (routed experts split over the ranks)",
            "value": world * T / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg["dtype"],
            "data": "synthetic (seeded counter-based generator; random-init weights)",
            "config": {"workload": args.config, "T_per_gpu": T, "D": D, "M": cfg["M"], "k": cfg["k"],
                       "I": cfg["I"], "I_sh": cfg.get("I_sh", 0), "parallelism": f"ep{world}",
                       "l2": "flushed between steps (256 MiB write outside the timed events)"},
            "exchange": {"capacity_factor": args.capacity_factor, "cap_rows_per_expert_per_rank": bufs["cap"],
                         "rows_per_rank_pair": bufs["R"] // world,
                         "pairs_kept_rank0": kept_sent, "pairs_dropped_rank0": T * cfg["k"] - kept_sent,
                         "rows_received_rank0": kept_recv,
                         "bytes_out_per_rank": (world - 1) * (bufs["R"] // world) * (
                             D * (2 if cfg["dtype"] == "bf16" else 4) + 4 + D * 4)},
            "e2e": None, "gpu_launches": launches, "gpu_launches_note": "rank 0's own kernels; NCCL's not counted",
            "clocks": clocks,
        }
        print(json.dumps(out), flush=True)
    del layer
    if dist is not None:
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.ep:
        run_ep(args)
    elif args.which == "backward":
        run_backward(args)
    elif is_dense(workload_config(args)):
        run_dense(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
