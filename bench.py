#!/usr/bin/env python
"""Throughput of the top-k softmax-routed latent MoE-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one moe_layer_forward over one batch of synthetic tokens: route, latent
down-projection, dispatch, expert gate/up and down GEMMs, normalise + combine, latent
up-projection with the residual gate.  Rank 0 prints one JSON line.

* value: tokens/s over all ranks (each rank processes the full workload: weak scaling, no
  data-path collective), from CUDA events around K steps, max over ranks;
* e2e: the same through the host-memory API (pinned host input -> device -> layer -> host, one
  pipelined moe_layer_forward_host call over the steps);
* ms_p50 / ms_p90: the median and 90th percentile of the per-step times of that timed region
  (an event between consecutive steps);
* roofline: the dominant kernel (expert gate/up GEMM) timed live with the library's stage events,
  in a second pass of K steps (the headline pass runs the layer without them);
* cpu_baseline: the CPU oracle on a bounded token sample of the same workload (rank 0, N=1);
* decode: the T=64 Muse decode workload measured the same way (secondary line item).

--impl reference times the CPU oracle (the only reference this path has) on the same workload,
metric and unit, a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

METRIC = "MoE-layer tokens/s (Muse shape, T=64 & T=16K) and % of HBM/BF16 roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "muse_prefill"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-decode", action="store_true", help="skip the secondary decode item")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=0, help="tokens in the CPU oracle sample")
    ap.add_argument("--expert-parallel", action="store_true",
                    help="run the workload expert-parallel over the ranks (NCCL all-to-all): each "
                         "rank holds n_experts / N experts and its own T tokens")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("at least 3 warm-up steps")
    return a


# ------------------------------------------------------------------ ranks

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init_dist(backend: str):
    import datetime
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def reduce_max(x: float, device=None) -> float:
    """Max of a float over ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks during the timed region

class ClockSampler:
    """nvidia-smi sampling every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        return self.parse(open(self.path).read())

    @staticmethod
    def parse(text: str) -> dict:
        sm, mx, reasons, power = [], [], set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in text.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx),
                "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


class NvmlClockSampler:
    """Reads the SM clock, power and clock-event reasons of one GPU every 20 ms through NVML
    (read-only queries) on a background thread while the timed region runs."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index: int):
        import threading
        import pynvml
        import torch
        self.nv = pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(device_index)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        self.samples = []
        self.stop_evt = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, pw, rs))
            except nv.NVMLError:
                pass
            self.stop_evt.wait(0.02)

    def start(self):
        self.thread.start()

    def stop(self) -> dict:
        self.stop_evt.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        reasons = set()
        for _, _, rs in self.samples:
            for name, const in self.REASONS:
                if rs & getattr(self.nv, const):
                    reasons.add(name)
        sm = [s for s, _, _ in self.samples]
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": self.max_mhz,
                "power_w_median": round(statistics.median(p for _, p, _ in self.samples), 1),
                "power_w_max": round(max(p for _, p, _ in self.samples), 1),
                "samples": len(self.samples), "source": "nvml 20 ms", "reasons": sorted(reasons)}


def make_sampler(local: int):
    try:
        return NvmlClockSampler(local)
    except Exception:  # no NVML: fall back to nvidia-smi sampling
        return ClockSampler(visible_gpu_index(local))


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ measured DRAM traffic

# DRAM bytes (read + write) per launch of the expert gate/up GEMM from one ncu capture of each
# reduced-expert case (32 experts at the full workload's rows per expert), with the units it
# processed.  A full
# launch scales by the same units: prefill by routed rows and experts (both 8x), decode by routed
# experts.  Valid only for the kernel source the capture was taken on (fingerprint below).
TRAFFIC_CAPTURES = {
    "kernel_sha256_16": "e59c35af08759c4a",
    "muse_prefill": {"bytes": 2.322391e9 + 0.130761216e9, "experts": 32, "rows": 2048 * 8},
    "muse_decode": {"bytes": 1.947448e9 + 0.004316416e9, "experts": 29, "rows": 8 * 8},
}


def kernel_fingerprint() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("common.cuh", "gemm_tc.cuh"):
        with open(os.path.join(ROOT, "sparse_moe_layer_softmax_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def gate_up_traffic(cfg, distinct_experts: int):
    """Measured traffic scaled to this launch, or None if the kernel changed since the capture."""
    cap = TRAFFIC_CAPTURES.get(cfg.name)
    if cap is None or kernel_fingerprint() != TRAFFIC_CAPTURES["kernel_sha256_16"]:
        return None
    if cfg.name == "muse_prefill":
        return round(cap["bytes"] * (cfg.T * cfg.top_k) / cap["rows"])
    return round(cap["bytes"] * distinct_experts / cap["experts"])


# ------------------------------------------------------------------ algorithmic work

def work_model(cfg, distinct_experts: int) -> dict:
    """Algorithmic FLOPs and HBM bytes of one layer forward and of its expert gate/up GEMM:
    the contractions the method must do, the weights it must read (only the distinct experts
    routed), the input read once and the output written once; intermediates that a fused
    design could keep on chip are not counted."""
    T, d, n, k, H = cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff
    E = cfg.expert_in
    b = 2 if cfg.dtype == "bf16" else 4
    gu = cfg.gu_rows
    expert_w = gu * E + E * H                      # elements of one expert's two matrices
    flops = 2 * T * (d * n + k * expert_w)
    wbytes = n * d * (4 if cfg.router_f32 else b) + distinct_experts * expert_w * b
    if cfg.latent:
        flops += 2 * T * (d * cfg.d_latent * 2)
        wbytes += 2 * cfg.d_latent * d * b
    act_bytes = 2 * T * d * b                       # u in, out back
    gate_up = {"flops": 2 * T * k * E * gu,
               "bytes": distinct_experts * gu * E * b + T * k * E * b + T * k * H * b}
    experts = {"flops": 2 * T * k * expert_w,                      # the routed experts alone
               "bytes": distinct_experts * expert_w * b + 2 * T * k * E * b}
    return {"flops": flops, "bytes": wbytes + act_bytes, "gate_up": gate_up, "experts": experts}


def roofline_entry(bound: str, work: float, seconds: float, peaks: dict, sustained: bool,
                   traffic=None) -> dict:
    if bound == "tensor":
        peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
        achieved = work / seconds / 1e12
        unit = "TFLOP/s"
    else:
        peak = peaks["hbm_gbs"]
        achieved = work / seconds / 1e9
        unit = "GB/s"
    return {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": peaks["source"] + (" sustained" if sustained and bound == "tensor"
                                              else "")}


# ------------------------------------------------------------------ our arm

def measure_ours(cfg, steps: int, warmup: int, device, peaks: dict, with_e2e: bool = True,
                 sampler=None) -> dict:
    import torch
    import moe_inputs
    import sparse_moe_layer_softmax_b200 as moe
    from gpu_harness import abi_config

    dev = moe_inputs.device_inputs(cfg, device=device)
    layer = moe.MoELayer(abi_config(cfg), dev)
    u = dev["u"]
    out = torch.empty_like(u)
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        layer.forward(u, u, out=out, topk_idx_out=idx)
    status = moe.moe_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status {moe.STATUS.get(status, status)} after warm-up")
    distinct = int(torch.unique(idx).numel())
    loads = torch.bincount(idx.flatten().long(), minlength=cfg.n_experts)
    max_over_mean = float(loads.max().item()) / (cfg.T * cfg.top_k / cfg.n_experts)

    # ---- device-resident timed region: the plain layer (no stage events inside a forward); an
    # event between consecutive steps gives each step's duration as well as the total
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    launches0 = moe.launch_count()
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    marks[0].record(stream)
    for i in range(steps):
        layer.forward(u, u, out=out, topk_idx_out=idx)
        marks[i + 1].record(stream)
    torch.cuda.synchronize()
    launches = moe.launch_count() - launches0
    clocks = sampler.stop() if sampler else None
    barrier()
    per_step = [marks[i].elapsed_time(marks[i + 1]) for i in range(steps)]
    ms = marks[0].elapsed_time(marks[steps]) / steps
    ms_max = reduce_max(ms, device)
    p50 = reduce_max(float(np.percentile(per_step, 50)), device)
    p90 = reduce_max(float(np.percentile(per_step, 90)), device)
    step_range = (round(min(per_step), 4), round(max(per_step), 4))
    status = moe.moe_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status {moe.STATUS.get(status, status)} after timing")

    # ---- stage breakdown in a pass of its own: the library's per-stage events around each stage
    moe.profile_begin(steps)
    for _ in range(steps):
        layer.forward(u, u, out=out, topk_idx_out=idx)
    torch.cuda.synchronize()
    stage_ms, calls = moe.profile_end()

    work = work_model(cfg, distinct)
    gate_up_s = stage_ms["expert_gate_up"] / max(calls, 1) / 1e3
    tensor_bound = work["flops"] / (peaks["bf16_tflops_sustained"] * 1e12) > \
        work["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if tensor_bound:
        roof = roofline_entry("tensor", work["gate_up"]["flops"], gate_up_s, peaks, True)
    else:
        roof = roofline_entry("hbm", work["gate_up"]["bytes"], gate_up_s, peaks, False)
    roof["traffic"] = gate_up_traffic(cfg, distinct)
    roof["algorithmic_bytes"] = work["gate_up"]["bytes"]
    roof["kernel"] = "expert gate/up GEMM (gemm_tc_kernel, SwiGLU epilogue)"
    roof["ms_per_launch"] = round(gate_up_s * 1e3, 4)
    t_roof = max(work["flops"] / (peaks["bf16_tflops_sustained"] * 1e12),
                 work["bytes"] / (peaks["hbm_gbs"] * 1e9))
    t_exp = max(work["experts"]["flops"] / (peaks["bf16_tflops_sustained"] * 1e12),
                work["experts"]["bytes"] / (peaks["hbm_gbs"] * 1e9))
    res = {"ms_per_step": ms_max, "ms_p50": round(p50, 4), "ms_p90": round(p90, 4),
           "ms_min_max": step_range,
           "tokens_per_step": cfg.T, "roofline": roof,
           "layer_roofline": {"bound": "tensor" if tensor_bound else "hbm",
                              "flops": work["flops"], "bytes": work["bytes"],
                              "roofline_ms": round(t_roof * 1e3, 4),
                              "frac": round(t_roof * 1e3 / ms_max, 4),
                              # the metric's literal reading: only the routed experts' work
                              # (router and latent projections excluded), against the same step
                              "experts_only_roofline_ms": round(t_exp * 1e3, 4),
                              "experts_only_frac": round(t_exp * 1e3 / ms_max, 4)},
           "stage_ms": {k: round(v / max(calls, 1), 4) for k, v in stage_ms.items()},
           "distinct_experts": distinct, "max_over_mean_load": round(max_over_mean, 3),
           "gpu_launches": int(launches), "clocks": clocks}

    # ---- end to end through the host-memory API: pinned host in, pinned host out.  One call
    # streams `steps` batches; every batch's input copy and output copy is inside the timed
    # region (the library overlaps them with the neighbouring batches' kernels).
    if with_e2e:
        u_host = u.cpu().pin_memory()
        out_host = torch.empty_like(u_host).pin_memory()
        layer.forward_host([u_host] * 2, [out_host] * 2, stream=stream)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer.forward_host([u_host] * steps, [out_host] * steps, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        res["e2e_ms"] = reduce_max(e0.elapsed_time(e1) / steps, device)
        res["h2d_bytes"] = u_host.numel() * u_host.element_size()
        res["d2h_bytes"] = out_host.numel() * out_host.element_size()
    del layer, dev
    torch.cuda.empty_cache()
    return res


def measure_gate_stats(cfg, args, device) -> dict:
    """moe_noisy_gate (noisy logits, KeepTopK gate, importance and smooth load with CV^2) on one
    batch, timed with CUDA events over the steps."""
    import torch
    import moe_inputs
    import sparse_moe_layer_softmax_b200 as moe
    from gpu_harness import abi_config
    dev = moe_inputs.device_inputs(cfg, device=device)
    c = abi_config(cfg)
    args_ = (c, dev["u"], dev["w_router"], dev["w_noise"], dev["noise_eps"])
    # the same call as timed, so that the allocator's cache holds every buffer size it asks for;
    # only the last call's outputs stay alive
    out = None
    for _ in range(args.warmup):
        out = moe.noisy_gate(*args_, want_h=False, want_p=False)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        out = moe.noisy_gate(*args_, want_h=False, want_p=False)
    e1.record()
    torch.cuda.synchronize()
    ms = reduce_max(e0.elapsed_time(e1) / args.steps, device)
    cv2 = out["cv2"].cpu().tolist()
    del dev, out
    torch.cuda.empty_cache()
    return {"value": round(cfg.T / (ms / 1e3), 2), "unit": UNIT, "ms_per_step": round(ms, 4),
            "cv2_importance": cv2[0], "cv2_load": cv2[1],
            "note": "includes the allocation of each call's outputs and workspace by the binding"}


def measure_graph(cfg, args, device, peaks: dict) -> dict:
    """The layer forward captured once in a CUDA graph and replayed K times (the host's launch
    work leaves the step); CUDA events around the replays."""
    import torch
    import moe_inputs
    import sparse_moe_layer_softmax_b200 as moe
    from gpu_harness import abi_config
    dev = moe_inputs.device_inputs(cfg, device=device)
    layer = moe.MoELayer(abi_config(cfg), dev)
    u = dev["u"]
    out = torch.empty_like(u)
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device=device)
    for _ in range(args.warmup):
        layer.forward(u, u, out=out, topk_idx_out=idx)
    torch.cuda.synchronize()
    distinct = int(torch.unique(idx).numel())
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        layer.forward(u, u, out=out)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(e0.elapsed_time(e1) / args.steps, device)
    status = moe.moe_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status {moe.STATUS.get(status, status)}")
    work = work_model(cfg, distinct)
    t_roof = max(work["flops"] / (peaks["bf16_tflops_sustained"] * 1e12),
                 work["bytes"] / (peaks["hbm_gbs"] * 1e9))
    del g, layer, dev
    torch.cuda.empty_cache()
    return {"value": round(cfg.T / (ms / 1e3), 2), "unit": UNIT, "ms_per_step": round(ms, 4),
            "layer_roofline": {"roofline_ms": round(t_roof * 1e3, 4),
                               "frac": round(t_roof * 1e3 / ms, 4)},
            "note": "one forward captured in a CUDA graph, replayed K times"}


def ep_ranks(cfg, world: int, device, rank_ids=None):
    """Expert-parallel ranks of `cfg` (cfg.T tokens per rank): rank r holds experts
    expert_ranges(n, world)[r] of the whole layer's weights, and tokens [r T, (r+1) T) of a
    world x T batch.  Returns (ranks, us) for rank_ids (all ranks by default)."""
    import moe_inputs
    from gpu_harness import abi_config
    from sparse_moe_layer_softmax_b200 import expert_parallel as ep
    dev = moe_inputs.device_inputs(cfg.replace(T=cfg.T * world), device=device)
    ranges = ep.expert_ranges(cfg.n_experts, world)
    ranks, us = [], []
    for r in (range(world) if rank_ids is None else rank_ids):
        lo, hi = ranges[r]
        w = {k: v for k, v in dev.items() if k not in ("u", "w_gu", "w_down")}
        w["w_gu"] = dev["w_gu"][lo:hi].clone()
        w["w_down"] = dev["w_down"][lo:hi].clone()
        ranks.append(ep.ExpertParallelRank(abi_config(cfg), w, r, world))
        us.append(dev["u"][r * cfg.T:(r + 1) * cfg.T].clone())
    del dev
    return ranks, us


def measure_ep_emulated(cfg, world: int, args, device, peaks: dict) -> dict:
    """The compute of one rank of a `world`-GPU expert-parallel layer (cfg.T tokens per rank),
    with every rank run on this GPU (the exchanges become slicing and concatenation).  Each stage
    of each rank is timed with CUDA events; a rank's step is its dispatch + its experts' compute
    on the rows all ranks sent it + its finish, and the slowest rank sets the step.  The NVLink
    exchange is not measured: its lower bound is the rows each rank sends and receives over the
    measured peer-copy bandwidth."""
    import torch
    from sparse_moe_layer_softmax_b200 import expert_parallel as ep
    ranks, us = ep_ranks(cfg, world, device)
    stream = torch.cuda.current_stream()
    log = []

    def timer(stage, r, fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        out = fn()
        b.record(stream)
        log.append((stage, r, a, b))
        return out
    for _ in range(args.warmup):
        ep.emulated_forward(ranks, us)
    torch.cuda.synchronize()
    per_step = []
    sent = []
    for _ in range(args.steps):
        log.clear()
        ep.emulated_forward(ranks, us, timer=timer)
        torch.cuda.synchronize()
        t = np.zeros((3, world))
        for stage, r, a, b in log:
            t[("dispatch", "compute", "finish").index(stage), r] += a.elapsed_time(b)
        per_step.append(t)
    t = np.mean(per_step, axis=0)
    rank_ms = t.sum(0)
    # rows a rank sends to the other ranks (and receives back), one bf16 row of E_in each way
    E = cfg.d_latent or cfg.d_model
    xfer = cfg.T * cfg.top_k * (world - 1) / world * E * 2 * 2
    link = 770e9
    ms = float(rank_ms.max())
    del ranks, us
    torch.cuda.empty_cache()
    return {"ranks": world, "tokens_per_rank": cfg.T,
            "value_compute_only": round(cfg.T * world / (ms / 1e3), 2), "unit": UNIT,
            "rank_compute_ms": round(ms, 4),
            "stage_ms_max_over_ranks": {"dispatch": round(float(t[0].max()), 4),
                                        "experts": round(float(t[1].max()), 4),
                                        "finish": round(float(t[2].max()), 4)},
            "exchange_bytes_per_rank": int(xfer),
            "exchange_floor_ms": round(xfer / link * 1e3, 4),
            "note": "one GPU runs every rank; times include each stage's host bookkeeping (the "
                    "dispatch reads its expert counts back); the NVLink exchange is not measured "
                    "(floor at the measured 770 GB/s peer copy)"}


def measure_ep_dist(cfg, args, device, rank: int, world: int) -> dict:
    """One rank of a real expert-parallel layer over torch.distributed (NCCL all-to-all between
    the GPUs): cfg.T tokens and n_experts / world experts on each rank.  CUDA events around the
    steps, max over ranks."""
    import torch
    from sparse_moe_layer_softmax_b200 import expert_parallel as ep
    (er,), (u,) = ep_ranks(cfg, world, device, rank_ids=[rank])
    exchange, counts = ep.dist_exchange(), ep.dist_exchange_counts(world)
    for _ in range(args.warmup):
        ep.forward(er, u, exchange, counts)
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        ep.forward(er, u, exchange, counts)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = reduce_max(e0.elapsed_time(e1) / args.steps, device)
    import sparse_moe_layer_softmax_b200 as moe
    status = moe.moe_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status {moe.STATUS.get(status, status)}")
    return {"ms_per_step": ms}


# ------------------------------------------------------------------ the CPU oracle as a baseline

class OracleRunner:
    """The CPU oracle on sampled tokens of a workload.  Weights are generated on the host once
    (they are the layer's parameters, resident like the GPU's); each run routes, evaluates the
    experts and projects the listed tokens with the oracle's own threads."""

    def __init__(self, cfg):
        import moe_inputs
        self.cfg = cfg
        self.dense = {name: moe_inputs.host_rows(cfg, name) for name in moe_inputs.tensor_specs(cfg)
                      if name not in ("u", "w_gu", "w_down")}
        if cfg.zipf_bias:
            self.dense["logit_bias"] = moe_inputs.zipf_bias(cfg)
        self.experts = {}

    def _inputs(self, tokens):
        import moe_inputs
        d = dict(self.dense)
        d["u"] = moe_inputs.host_rows(self.cfg, "u", rows=tokens)
        return d

    def _expert(self, e):
        import moe_inputs
        if e not in self.experts:
            self.experts[e] = (moe_inputs.host_rows(self.cfg, "w_gu", lead=e),
                               moe_inputs.host_rows(self.cfg, "w_down", lead=e))
        return self.experts[e]

    def prepare(self):
        """Untimed: generate the host weights of every expert."""
        for e in range(self.cfg.n_experts):
            self._expert(e)

    def run(self, tokens) -> float:
        """Seconds of wall time for the oracle on these tokens."""
        import oracle
        t0 = time.perf_counter()
        oracle.layer_forward_staged(self.cfg, tokens, self._inputs, self._expert)
        return time.perf_counter() - t0


def cpu_sample_tokens(cfg, count: int, salt: int = 0):
    import moe_inputs
    from moe_inputs import configs
    toks = moe_inputs.fisher_yates(cfg.seed + 1000 * (salt + 1), configs.STREAM_SUBSAMPLE,
                                   cfg.T, count)
    return np.sort(toks)


def default_cpu_sample(cfg) -> int:
    """Tokens per CPU-oracle sample: about 10-30 s of work on the host's cores."""
    per_token_gmac = (cfg.d_model * cfg.n_experts + cfg.top_k * (cfg.gu_rows * cfg.expert_in +
                      cfg.expert_in * cfg.d_ff) + 2 * cfg.d_model * cfg.d_latent) / 1e9
    cores = os.cpu_count() or 1
    # the staged double-precision oracle does about 0.08 GMAC/s per core (measured: 127 prefill
    # tokens in 46 s on 16 threads)
    n = int(15.0 * cores * 0.08 / max(per_token_gmac, 1e-6))
    return int(max(cores, min(n, cfg.T, 4096)))


def cpu_baseline(cfg, sample: int) -> dict:
    runner = OracleRunner(cfg)
    toks = cpu_sample_tokens(cfg, sample)
    runner.prepare()
    secs = runner.run(toks)
    return {"value": round(len(toks) / secs, 3), "unit": UNIT, "cores": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{len(toks)} seeded tokens of {cfg.name} (T={cfg.T}); full layer per token "
                      f"in double on {os.cpu_count()} threads; host weights generated untimed",
            "seconds": round(secs, 3)}


def config_block(cfg, world: int) -> dict:
    return {"workload": cfg.name, "T": cfg.T, "d_model": cfg.d_model, "d_latent": cfg.d_latent,
            "d_ff": cfg.d_ff, "n_experts": cfg.n_experts, "top_k": cfg.top_k, "seed": cfg.seed,
            "global_batch": cfg.T * world,
            "separated_inputs": {"redrawn_tokens": len(cfg.u_redraw),
                                 "separation": "top-k margin >= 1e-3 rms of the router keys"},
            "parallelism": f"replicas x{world}: every rank runs the full workload",
            "l2": "no flush: every step streams the routed experts' weights (GBs) and activations "
                  "far larger than the 126 MB L2"}


# ------------------------------------------------------------------ reference arm: the CPU oracle

def run_reference(args) -> int:
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from moe_inputs import configs
    cfg = configs.ALL_CONFIGS[args.workload]
    runner = OracleRunner(cfg)
    runner.prepare()
    per_step = args.cpu_sample or (os.cpu_count() or 1)
    for s in range(args.warmup):
        runner.run(cpu_sample_tokens(cfg, per_step, salt=100 + s))
    secs = 0.0
    for s in range(args.steps):
        secs += runner.run(cpu_sample_tokens(cfg, per_step, salt=s))
    value = per_step * args.steps / secs
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg, 1),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": os.cpu_count(),
                             "kind": "oracle",
                             "sample": f"{per_step} seeded tokens of {cfg.name} per step"},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main

def visible_gpu_index(local: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def measure_checked(cfg, args, device, peaks, rank, local, with_e2e=True) -> dict:
    """Measure; re-measure once if the clocks record shows a rejected throttle reason."""
    for attempt in range(2):
        sampler = make_sampler(local) if rank == 0 else None
        res = measure_ours(cfg, args.steps, args.warmup, device, peaks, with_e2e, sampler)
        clk = res.get("clocks") or {}
        bad = BAD_REASONS & set(clk.get("reasons") or [])
        if not bad:
            break
        res["remeasured_after"] = sorted(bad)
    return res


def main_expert_parallel(cfg, args, device, rank: int, world: int) -> int:
    """bench.py --expert-parallel: the layer expert-parallel over the ranks."""
    import datetime
    import socket
    import torch.distributed as dist
    if not dist.is_initialized():
        # one rank: a one-member NCCL group, so that the same all-to-all path runs
        with socket.socket() as s_:
            s_.bind(("127.0.0.1", 0))
            port = s_.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120))
    res = measure_ep_dist(cfg, args, device, rank, world)
    if rank == 0:
        block = config_block(cfg, world)
        block["parallelism"] = (f"expert parallel x{world}: each rank holds {cfg.n_experts // world} "
                                f"experts and routes its own {cfg.T} tokens; NCCL all-to-all "
                                "dispatch and return")
        line = {"metric": METRIC, "value": round(cfg.T * world / (res["ms_per_step"] / 1e3), 2),
                "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(res["ms_per_step"], 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded counter-based generator; random-init weights)",
                "config": block}
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None) -> int:
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    import torch
    from moe_inputs import configs
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist("nccl")
    peaks = measured_peaks()
    cfg = configs.ALL_CONFIGS[args.workload]
    if args.expert_parallel:
        return main_expert_parallel(cfg, args, device, rank, world)
    res = measure_checked(cfg, args, device, peaks, rank, local)
    value = cfg.T * world / (res["ms_per_step"] / 1e3)
    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(res["ms_per_step"], 4),
            "ms_p50": res["ms_p50"], "ms_p90": res["ms_p90"], "ms_min_max": res["ms_min_max"],
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded counter-based generator; random-init weights)",
            "config": config_block(cfg, world),
            "roofline": res["roofline"], "layer_roofline": res["layer_roofline"],
            "e2e": {"value": round(cfg.T * world / (res["e2e_ms"] / 1e3), 2), "unit": UNIT,
                    "h2d_bytes_per_step": res["h2d_bytes"], "d2h_bytes_per_step": res["d2h_bytes"],
                    "ms_per_step": round(res["e2e_ms"], 4)},
            "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
            "stage_ms": res["stage_ms"], "distinct_experts": res["distinct_experts"],
            "max_over_mean_load": res["max_over_mean_load"]}
    if "remeasured_after" in res:
        line["remeasured_after"] = res["remeasured_after"]
    if not args.no_decode and cfg.name != "muse_decode":
        dres = measure_checked(configs.MUSE_DECODE, args, device, peaks, rank, local)
        line["decode"] = {
            "workload": "muse_decode", "value": round(64 * world / (dres["ms_per_step"] / 1e3), 2),
            "unit": UNIT, "ms_per_step": round(dres["ms_per_step"], 4),
            "ms_p50": dres["ms_p50"], "ms_p90": dres["ms_p90"], "roofline": dres["roofline"], "layer_roofline": dres["layer_roofline"],
            "e2e": {"value": round(64 * world / (dres["e2e_ms"] / 1e3), 2), "unit": UNIT,
                    "h2d_bytes_per_step": dres["h2d_bytes"],
                    "d2h_bytes_per_step": dres["d2h_bytes"]},
            "stage_ms": dres["stage_ms"], "distinct_experts": dres["distinct_experts"],
            "gpu_launches": dres["gpu_launches"], "clocks": dres["clocks"]}
    if not args.no_decode and cfg.name != "muse_decode":
        # decode with the Muse router as the Muse audit describes it (fp32 weights, sigmoid
        # gate), and the decoder layer's whole FFN sub-block (input norm, output norm)
        line["variants"] = {}
        for vcfg in (configs.MUSE_DECODE_SIGMOID, configs.MUSE_DECODE_BLOCK,
                     configs.SHAZEER_BF16, configs.MUSE_IMBALANCED):
            vres = measure_checked(vcfg, args, device, peaks, rank, local, with_e2e=False)
            line["variants"][vcfg.name] = {
                "value": round(vcfg.T * world / (vres["ms_per_step"] / 1e3), 2), "unit": UNIT,
                "ms_per_step": round(vres["ms_per_step"], 4), "ms_p50": vres["ms_p50"],
                "ms_p90": vres["ms_p90"], "stage_ms": vres["stage_ms"],
                "layer_roofline": vres["layer_roofline"], "clocks": vres["clocks"]}
    if not args.no_decode and cfg.name != "muse_decode":
        line["variants"]["muse_decode_cuda_graph"] = measure_graph(configs.MUSE_DECODE, args,
                                                                   device, peaks)
    if not args.no_decode and cfg.name != "muse_decode":
        line.setdefault("variants", {})["shazeer_bf16_noisy_gate_stats"] = measure_gate_stats(
            configs.SHAZEER_BF16_NOISY, args, device)
    if not args.no_decode and world == 1:
        # the decode workload as one rank of an 8-GPU expert-parallel layer (64 tokens and 32
        # experts per rank), every rank emulated on this GPU: the ranks' compute only
        line.setdefault("variants", {})["muse_decode_ep8_emulated"] = measure_ep_emulated(
            configs.MUSE_DECODE, 8, args, device, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_sample or default_cpu_sample(cfg))
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

