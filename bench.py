#!/usr/bin/env python
"""Benchmark of one sparse MoE layer forward over FP4 experts on B200.

Metric: MoE-layer tokens/s.  Default workload (the largest single-GPU layer):
the Qwen3.8-Flash-Next-like layer (hidden 4096, expert intermediate 1024, 512
NVFP4 experts, top-10 plus one bf16 shared expert, Zipf-skewed routing) at a
prefill of 8192 tokens with its own resident budget of 46 of 512 experts
(hottest first), the rest copied from pinned host memory, EXACT numerics.  A
step is one full layer forward (router, top-k, permutation, misses staged from
host memory, expert gate/up + SwiGLU, down + gate scale, shared expert,
combine) of one batch.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME --tokens T]
  python bench.py --impl reference ...   # the CPU oracle arm (rank 0 only)

Besides the headline line, the same run measures (unless --no-legs):
  * the binding roof tau = max(t_HBM, t_PCIe, t_TC) + serial, with the pinned
    host-to-device bandwidth measured in this process;
  * the same layer all resident (the prefill kernels' own roofline);
  * the OLMoE-like decode step (32 tokens, HBM roofline of the gate/up pass);
  * the compute-bound A4 probe (FP4 tensor-pipe fraction of the FP4 GEMM).

Multi-GPU: one process per GPU (torchrun), each rank an independent replica on
its own batch (the layer has no exchange step), so value = all tokens / max
rank time and scaling is weak.

Timing: per step, L2 is flushed (a 256 MiB write) outside the timed events,
then CUDA events on the launching stream bracket the forward; the timed region
is bracketed by a barrier and device synchronisation and the result is the
maximum over ranks.  Stage timing (CUDA events recorded by the library around
each kernel, in a separate pass) gives the live duration of the dominant
kernel for the roofline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
METRIC = "MoE-layer tokens/s on 1 B200; % HBM roofline (decode), % FP4 peak (prefill)"
DEFAULT_WORKLOAD = "qwen3_8_flash_next_like"


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    p.add_argument("--tokens", type=int, default=None,
                   help="batch size (default: the workload's prefill size, else its largest decode batch)")
    p.add_argument("--numerics", default="exact", choices=["exact", "a4"])
    p.add_argument("--slots", default="workload", choices=["workload", "all"],
                   help="resident budget: the workload's own, or every expert resident")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU baseline sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay leg")
    p.add_argument("--no-legs", action="store_true", help="skip the resident / decode / FP4-probe legs")
    a = p.parse_args(argv)
    if a.tokens is None:
        wl = synth.workload(a.workload)
        a.tokens = wl.prefill_tokens or max(wl.decode_tokens)
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.idx = device_index

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.idx is not None:
            cmd += ["-i", self.idx]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def pci_index(torch, dev):
    try:
        pr = torch.cuda.get_device_properties(dev)
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except Exception:
        return None


# ------------------------------------------------------------------ work model
def gateup_bytes(wl, n_active, T):
    """Algorithmic HBM bytes of one routed gate/up launch: the gate and up codes and
    block scales of every active expert, the activations read once, and h written."""
    per_expert = 2 * wl.inter * wl.hidden * (0.5 + 1.0 / wl.group)
    return n_active * per_expert + T * wl.hidden * 2 + T * wl.top_k * wl.inter * 2


def layer_bytes(wl, n_active, T):
    """Algorithmic HBM bytes of one forward (unique active experts read once + router +
    shared expert + x + y)."""
    b = n_active * wl.expert_bytes() + wl.n_experts * wl.hidden * 4 + T * wl.hidden * (2 + 4)
    if wl.shared_inter:
        b += 3 * wl.shared_inter * wl.hidden * 2
    return b


def routed_flops(wl, T):
    """Multiply-add FLOPs of the routed experts (gate, up and down) for T tokens."""
    return 6.0 * T * wl.top_k * wl.hidden * wl.inter


def gateup_flops(wl, T):
    return 4.0 * T * wl.top_k * wl.hidden * wl.inter


def shared_flops(wl, T):
    return 6.0 * T * wl.hidden * wl.shared_inter


def binding_roof(wl, T, n_active, miss_bytes, h2d_gbs, hbm_gbs, tensor_tflops, serial_ms, step_ms):
    """tau = max(t_HBM, t_PCIe, t_TC) + serial (the routing step and the combine,
    which no other stage can overlap), and the achieved fraction tau / step.

    t_HBM: algorithmic HBM bytes / measured copy bandwidth; t_PCIe: bytes of the
    experts staged from pinned host memory / measured pinned H2D bandwidth; t_TC:
    routed + shared FLOPs at `tensor_tflops` (the rate of the MMA kind the path
    uses)."""
    t_hbm = layer_bytes(wl, n_active, T) / (hbm_gbs * 1e9) * 1e3
    t_pcie = miss_bytes / (h2d_gbs * 1e9) * 1e3 if h2d_gbs else 0.0
    t_tc = (routed_flops(wl, T) + shared_flops(wl, T)) / (tensor_tflops * 1e12) * 1e3
    terms = {"t_hbm_ms": t_hbm, "t_pcie_ms": t_pcie, "t_tc_ms": t_tc}
    bind = max(terms, key=terms.get)
    tau = terms[bind] + serial_ms
    return {"tau_ms": tau, **terms, "serial_ms": serial_ms, "binding": bind[2:-3],
            "step_ms": step_ms, "frac_of_tau": tau / step_ms if step_ms > 0 else None}


def traffic_record(summary, kernel_src):
    """DRAM bytes per launch from a committed ncu summary (profiles/<summary>), if it
    was taken on the kernel source as it is now (its sha256 is recorded there)."""
    path = summary if os.path.isabs(summary) else os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    rec = {}
    with open(path) as f:
        for line in f:
            line = line.strip().lstrip("-* `")
            if ":" in line and line.startswith(("dram_bytes_per_launch", "kernel_source_sha256")):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip(" `")
    with open(kernel_src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    if rec.get("kernel_source_sha256") != h or "dram_bytes_per_launch" not in rec:
        return None
    return float(rec["dram_bytes_per_launch"])


# ------------------------------------------------------------------ CPU (oracle) legs
def cpu_baseline(lw, x_bits, budget_s, numerics="exact"):
    """The oracle as it stands, all host threads, forwards over consecutive
    slices of the benchmark batch (the whole batch when it is small) until the
    time budget is spent."""
    import oracle
    L = oracle.Layer.from_weights(lw, numerics=numerics)
    threads = oracle.max_threads()
    T = x_bits.shape[0]
    chunk = T if T <= 64 else max(2 * threads, 16)
    n, i, t0 = 0, 0, time.perf_counter()
    while True:
        c = min(chunk, T - i)
        L.forward(x_bits[i:i + c], threads=threads)
        n += c
        i = (i + c) % T
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    what = (f"full forwards of the {T}-token batch" if chunk == T
            else f"forwards of consecutive {chunk}-token slices of the {T}-token batch")
    return {"value": n / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{what} ({n} tokens, {el:.1f} s, {numerics} numerics)"}


def gpu_local_cpus(torch, dev_index, nvml=None):
    """The host CPUs NVML reports as local to this process's GPU (its NUMA
    node), intersected with the CPUs the process may run on; None when NVML
    cannot tell.  With one replica per GPU, each rank's pinned expert store
    and staging copies then sit on the socket its GPU hangs off."""
    try:
        if nvml is None:
            import pynvml as nvml
        nvml.nvmlInit()
        h = None
        props = torch.cuda.get_device_properties(dev_index) if torch is not None else None
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devn = getattr(props, "pci_device_id", 0)
            try:
                h = nvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devn:02x}.0")
            except Exception:
                h = None
        if h is None:
            h = nvml.nvmlDeviceGetHandleByIndex(dev_index)
        words = nvml.nvmlDeviceGetCpuAffinity(h, ((os.cpu_count() or 64) + 63) // 64)
        cpus = {64 * w + b for w, m in enumerate(words) for b in range(64) if (int(m) >> b) & 1}
    except Exception:
        return None
    local = cpus & os.sched_getaffinity(0)
    return local or None


def max_over_ranks(vals, world):
    """Element-wise maximum of this rank's timings over all ranks, returned on
    every rank: the job is as slow as its slowest replica."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    return vals


def whole_job_tokens_per_s(world, tokens_per_rank, steps, max_ms):
    """Tokens of all ranks (independent replicas, one batch each per step)
    over the slowest rank's time for `steps` steps."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


def reference_arm(args, wl, lw, world):
    """--impl reference: the oracle timed on host cores, each step a bounded sample."""
    import oracle
    L = oracle.Layer.from_weights(lw)
    T = args.tokens
    x = synth.make_tokens(wl, T)
    _, ids, _ = L.route_all(x)
    rows_per_token = wl.top_k * wl.inter
    t0 = time.perf_counter()
    L.expert_rows(int(ids[0, 0]), x[0], 0, 16)
    t_row = max((time.perf_counter() - t0) / 16, 1e-7)
    budget = 150.0
    rows = int(max(1, min(wl.inter, budget / ((args.steps + args.warmup) * t_row))))

    def step(i):
        t = i % T
        j = (i // T) % wl.top_k
        e = int(ids[t, j])
        i0 = (i * rows) % wl.inter
        n = min(rows, wl.inter - i0)
        L.expert_rows(e, x[t], i0, n)
        return n

    for i in range(args.warmup):
        step(i)
    done = 0
    t0 = time.perf_counter()
    for i in range(args.steps):
        done += step(args.warmup + i)
    el = time.perf_counter() - t0
    tokens = done / rows_per_token
    value = tokens / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no dataset or trained weights)",
        "config": {"workload": wl.name, "tokens": T, "hidden": wl.hidden, "inter": wl.inter,
                   "n_experts": wl.n_experts, "top_k": wl.top_k, "fmt": wl.fmt},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: {rows} of the {rows_per_token} expert rows of one token "
                                   f"(one routed expert's gate/up/down rows), single thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
def pinned_h2d_gbs(torch, dev, nbytes=512 << 20, reps=5):
    """Pinned host -> device bandwidth of one large cudaMemcpyAsync (the copy the
    staging of a missed expert issues), median over `reps`, CUDA events."""
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    out = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        out.append(nbytes / (a.elapsed_time(b) / 1e3) / 1e9)
    del src, dst
    return statistics.median(out)


def time_steps(torch, layer, x, y, T, K, W, flush, stream):
    """W untimed warm-up forwards, then K forwards each bracketed by CUDA events
    on the launching stream (L2 flushed before each); returns the summed device
    ms and the library's stage profile from a separate pass."""
    sp = stream.cuda_stream
    for _ in range(W):
        flush.zero_()
        layer.forward_ptr(x.data_ptr(), T, y.data_ptr(), sp)
    torch.cuda.synchronize()
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        ev0[i].record(stream)
        layer.forward_ptr(x.data_ptr(), T, y.data_ptr(), sp)
        ev1[i].record(stream)
    torch.cuda.synchronize()
    dev_ms = sum(a.elapsed_time(b) for a, b in zip(ev0, ev1))
    return dev_ms


def stage_profile(torch, layer, x, y, T, n, flush, stream):
    layer.profile_enable(True)
    for _ in range(n):
        flush.zero_()
        layer.forward_ptr(x.data_ptr(), T, y.data_ptr(), stream.cuda_stream)
    torch.cuda.synchronize()
    prof = layer.profile_read()
    layer.profile_enable(False)
    return prof


def per_step(prof, stage):
    return prof["ms"][stage] / max(1, prof["forwards"])


def gateup_roofline(wl, T, n_active, prof, hbm_peak, bf16_sus, numerics, peak_src, traffic=None):
    """Roofline of the routed gate/up pass (the dominant kernel): summed over the
    pass's launches in a step (one per staging wave when experts are paged)."""
    g_ms = per_step(prof, "gateup")
    launches = prof["launches"]["gateup"] / max(1, prof["forwards"])
    if numerics == "a4":
        flops = gateup_flops(wl, T)
        peak = 4.0 * bf16_sus
        ach = flops / (g_ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                "traffic": traffic, "kernel": "gemm_a4_kernel gate/up+SwiGLU (tcgen05 block-scaled FP4)",
                "peak_source": f"{peak_src} bf16_tflops_sustained x 4 (nominal FP4/BF16 dense ratio)",
                "algorithmic_flops_per_step": flops, "kernel_ms_per_step": g_ms, "launches_per_step": launches,
                "hbm_gbs_of_same_pass": gateup_bytes(wl, n_active, T) / (g_ms / 1e3) / 1e9}
    prefill_nv = wl.fmt == "nvfp4" and T * wl.top_k > 12 * min(wl.n_experts, T * wl.top_k)
    if prefill_nv:
        flops = gateup_flops(wl, T)
        ach = flops / (g_ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": bf16_sus, "unit": "TFLOP/s", "frac": ach / bf16_sus,
                "traffic": traffic,
                "kernel": "expert_dq_kernel gate/up+SwiGLU (tcgen05 kind::f16, NVFP4 decoded to f16 into TMEM as the A operand)",
                "peak_source": f"{peak_src} bf16_tflops_sustained (the MMA kind this path runs)",
                "algorithmic_flops_per_step": flops, "kernel_ms_per_step": g_ms, "launches_per_step": launches,
                "hbm_gbs_of_same_pass": gateup_bytes(wl, n_active, T) / (g_ms / 1e3) / 1e9}
    b = gateup_bytes(wl, n_active, T)
    ach = b / (g_ms / 1e3) / 1e9
    tc = wl.fmt == "mxfp4"
    return {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak,
            "traffic": traffic,
            "kernel": ("expert_tc_kernel gate/up+SwiGLU (tcgen05, E2M1 weights x E4M3 activation pieces)"
                       if tc else "expert_tma_kernel gate/up+SwiGLU (register decode, mma.sync)"),
            "peak_source": f"{peak_src} hbm_gbs", "algorithmic_bytes_per_step": b, "kernel_ms_per_step": g_ms,
            "launches_per_step": launches}


def short_leg(torch, F, dev, flush, stream, name, T, numerics, K, W, peaks_t, slots="all"):
    """One extra measurement on another workload / budget: tokens/s, step time
    and the gate/up pass's roofline."""
    hbm_peak, _, bf16_sus, src = peaks_t
    wl = synth.workload(name)
    lw = synth.make_layer(wl)
    S = wl.n_experts if slots == "all" else wl.n_slots
    layer = F.MoELayer.from_weights(lw, n_slots=S, max_tokens=T, numerics=numerics)
    try:
        layer.set_slot_table(synth.slot_table(lw, S))
        xb = synth.make_tokens(wl, T)
        x = torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((T, wl.hidden), dtype=torch.float32, device=dev)
        _, r = layer.forward(x, routing=True)
        torch.cuda.synchronize()
        n_active = int((r["counts"] > 0).sum().item())
        ms = time_steps(torch, layer, x, y, T, K, W, flush, stream) / K
        prof = stage_profile(torch, layer, x, y, T, min(K, 50), flush, stream)
        # DRAM bytes per gate/up launch from a committed ncu summary of the same
        # kernel source on the same workload (all resident: one launch per step)
        csrc = os.path.join(ROOT, "fp4_expert_layer_b200", "csrc")
        traffic = None
        if slots == "all" and numerics == "exact" and name == "olmoe_like" and T == 32:
            traffic = traffic_record("expert_tc_gateup_olmoe_like_T32.md", os.path.join(csrc, "expert_tc.cu"))
        elif slots == "all" and numerics == "exact" and name == "qwen3_8_flash_next_like" and T == 8192:
            traffic = traffic_record("expert_dq_gateup_qwen3_8_flash_next_like_T8192.md",
                                     os.path.join(csrc, "expert_dq.cu"))
        elif slots == "all" and numerics == "a4" and name == "fp4_peak_probe" and T == 8192:
            traffic = traffic_record("gemm_a4_gateup_fp4_peak_probe_T8192.md", os.path.join(csrc, "gemm_a4.cu"))
        roof = gateup_roofline(wl, T, n_active, prof, hbm_peak, bf16_sus, numerics, src, traffic)
        return {"workload": name, "tokens": T, "numerics": numerics, "resident_slots": S,
                "value": T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": K,
                "active_experts": n_active, "roofline": roof,
                "layer_hbm_frac": layer_bytes(wl, n_active, T) / (ms / 1e3) / 1e9 / hbm_peak,
                "stage_ms": {k: per_step(prof, k) for k in prof["ms"]}}
    finally:
        layer.close()


def main():
    args = parse()
    wl = synth.workload(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        if rank == 0:
            lw = synth.make_layer(wl)
            reference_arm(args, wl, lw, world)
        return

    import torch
    import torch.distributed as dist

    import fp4_expert_layer_b200 as F
    from fp4_expert_layer_b200 import build as fbuild

    if rank == 0:
        fbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    host_binding = "unchanged"
    if world > 1:
        # replicas: keep each rank's host memory and copy threads on its GPU's socket
        cpus = gpu_local_cpus(torch, local)
        if cpus:
            os.sched_setaffinity(0, cpus)
            host_binding = f"gpu-local cpus ({len(cpus)})"
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        dist.barrier()

    def barrier():
        if world > 1:
            dist.barrier()

    T = args.tokens
    lw = synth.make_layer(wl)
    S = wl.n_experts if args.slots == "all" else wl.n_slots
    layer = F.MoELayer.from_weights(lw, n_slots=S, max_tokens=T, numerics=args.numerics)
    layer.set_slot_table(synth.slot_table(lw, S))
    x_bits = synth.make_tokens(wl, T, stream=rank)
    x = torch.from_numpy(x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    y = torch.empty((T, wl.hidden), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    h2d_gbs = pinned_h2d_gbs(torch, dev)

    _, r = layer.forward(x, routing=True)
    torch.cuda.synchronize()
    n_active = int((r["counts"] > 0).sum().item())
    misses = int(layer.stats()["last_misses"])
    expert_bytes = int(layer.stats()["expert_bytes"])

    for _ in range(args.warmup):
        flush.zero_()
        layer.forward_ptr(x.data_ptr(), T, y.data_ptr(), sp)
    torch.cuda.synchronize()

    K = args.steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    clocks = ClockSampler(pci_index(torch, dev))
    launches0 = layer.stats()["launches"]
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for i in range(K):
        flush.zero_()
        ev0[i].record(stream)
        layer.forward_ptr(x.data_ptr(), T, y.data_ptr(), sp)
        ev1[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - w0
    clk = clocks.stop()
    launches = layer.stats()["launches"] - launches0
    dev_ms = sum(a.elapsed_time(b) for a, b in zip(ev0, ev1))
    # per-stage device times: a separate pass of the same loop with the
    # library's stage event pairs on, so that they do not touch the timed steps
    prof = stage_profile(torch, layer, x, y, T, min(K, 50), flush, stream)

    # e2e through the public host-buffer call: H2D of x, forward, D2H of y
    e2e = None
    if not args.no_e2e:
        xh = torch.from_numpy(x_bits.view(np.int16)).pin_memory()
        yh = torch.empty((T, wl.hidden), dtype=torch.float32).pin_memory()
        Ke = max(5, K // 4)
        for _ in range(2):
            layer.forward_host_ptr(xh.data_ptr(), T, yh.data_ptr(), sp)
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(Ke)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(Ke)]
        barrier()
        torch.cuda.synchronize()
        for i in range(Ke):
            flush.zero_()
            e0[i].record(stream)
            layer.forward_host_ptr(xh.data_ptr(), T, yh.data_ptr(), sp)
            e1[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = sum(a.elapsed_time(b) for a, b in zip(e0, e1))
        e2e = [e2e_ms, Ke]

    # CUDA-graph replay of the same forward (all-resident layers): the same
    # launch chain without the CPU cost of each launch; L2 flushed as above
    graph_ms = 0.0
    if S == wl.n_experts and not args.no_graph:
        gs = torch.cuda.Stream(dev)
        yg = torch.empty_like(y)
        gph = layer.capture_graph(x.data_ptr(), T, yg.data_ptr(), gs.cuda_stream)
        with torch.cuda.stream(gs):
            for _ in range(args.warmup):
                flush.zero_()
                gph.launch(gs.cuda_stream)
        gs.synchronize()
        g0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        g1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(gs):
            for i in range(K):
                flush.zero_()
                g0[i].record(gs)
                gph.launch(gs.cuda_stream)
                g1[i].record(gs)
        gs.synchronize()
        barrier()
        graph_ms = sum(a.elapsed_time(b) for a, b in zip(g0, g1))
        gph.close()
    layer.close()

    vals = torch.tensor([dev_ms, e2e[0] if e2e else 0.0, graph_ms], dtype=torch.float64, device=dev)
    vals = max_over_ranks(vals, world)
    dev_ms_max, e2e_ms_max, graph_ms_max = float(vals[0]), float(vals[1]), float(vals[2])

    # extra legs (every rank runs them, so that the collective sequence stays the same)
    pk = peaks()
    legs = {}
    if not args.no_legs and world == 1:
        if S < wl.n_experts:
            legs["resident_leg"] = short_leg(torch, F, dev, flush, stream, wl.name, T, args.numerics,
                                             max(5, K // 2), 2, pk)
        legs["decode_leg"] = short_leg(torch, F, dev, flush, stream, "olmoe_like", 32, "exact", 500, 20, pk)
        legs["fp4_leg"] = short_leg(torch, F, dev, flush, stream, "fp4_peak_probe", 8192, "a4", 20, 3, pk)

    if rank == 0:
        hbm_peak, bf16_peak, bf16_sus, peak_src = pk
        ms_step = dev_ms_max / K
        value = whole_job_tokens_per_s(world, T, K, dev_ms_max)
        roof = gateup_roofline(wl, T, n_active, prof, hbm_peak, bf16_sus, args.numerics, peak_src)
        serial = per_step(prof, "router") + per_step(prof, "permute") + per_step(prof, "combine")
        # A4: FP4 x FP4; EXACT: 4-bit weights times 16-bit activations run at the
        # bf16 rate (NVFP4: kind::f16) or as two 8-bit pieces at twice it (MXFP4)
        tensor_rate = 4.0 * bf16_sus if args.numerics == "a4" else bf16_sus
        roof["tau"] = binding_roof(wl, T, n_active, misses * expert_bytes, h2d_gbs, hbm_peak, tensor_rate,
                                   serial, ms_step)
        roof["tau"].update({"pinned_h2d_gbs_measured": h2d_gbs, "misses_per_step": misses,
                            "staged_bytes_per_step": misses * expert_bytes,
                            "tensor_rate_tflops": tensor_rate,
                            "tensor_rate_note": ("FP4 x FP4 at 4 x measured sustained bf16" if args.numerics == "a4"
                                                 else "EXACT numerics multiply 4-bit weights with 16-bit "
                                                      "activations: bf16 / 8-bit-piece tensor rate (measured "
                                                      "sustained bf16)"),
                            "serial_stages": "router + top-k + permutation, ordered combine"})
        stage_ms = {k: per_step(prof, k) for k in prof["ms"]}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": ("bf16xfp4->f32" if wl.fmt == "nvfp4" else "e4m3x2xfp4->f32")
            if args.numerics == "exact" else "fp4xfp4->f32",
            "data": "synthetic (seeded; random-init weights of the workload's shape)",
            "config": {"workload": wl.name, "tokens": T, "hidden": wl.hidden, "inter": wl.inter,
                       "n_experts": wl.n_experts, "top_k": wl.top_k, "fmt": wl.fmt,
                       "shared_inter": wl.shared_inter, "resident_slots": S, "numerics": args.numerics,
                       "parallelism": f"replicas x{world}", "l2": "flushed (256 MiB write) before every step",
                       "host_binding": host_binding,
                       "active_experts": n_active},
            "roofline": roof,
            "layer_roofline": {"bytes_per_step": layer_bytes(wl, n_active, T),
                               "hbm_frac": layer_bytes(wl, n_active, T) / (ms_step / 1e3) / 1e9 / hbm_peak},
            "stage_ms": stage_ms,
            "gpu_launches": int(launches),
            "wall_ms_per_step_incl_flush": 1e3 * wall / K,
            "clocks": clk,
        }
        if e2e:
            line["e2e"] = {"value": whole_job_tokens_per_s(world, T, e2e[1], e2e_ms_max), "unit": "tokens/s",
                           "h2d_bytes_per_step": T * wl.hidden * 2, "d2h_bytes_per_step": T * wl.hidden * 4}
        if graph_ms_max > 0:
            line["graph"] = {"value": whole_job_tokens_per_s(world, T, K, graph_ms_max), "unit": "tokens/s",
                             "ms_per_step": graph_ms_max / K,
                             "how": "moe_graph_capture of this forward, replayed K times (L2 flushed before each)"}
        line.update(legs)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(lw, x_bits, args.cpu_seconds, args.numerics)
        print(json.dumps(line), flush=True)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
