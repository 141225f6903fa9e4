#!/usr/bin/env python
"""Benchmark of one sparse MoE layer forward over FP4 experts on B200.

Metric: MoE-layer tokens/s.  Default workload: the OLMoE-like layer (hidden
2048, expert intermediate 1024, 64 MXFP4 experts, top-8, all resident) at a
decode batch of 32 tokens.  A step is one full layer forward (router, top-k,
permutation, expert gate/up + SwiGLU, down + gate scale, combine) of one batch.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME --tokens T]
  python bench.py --impl reference ...   # the CPU oracle arm (rank 0 only)

Multi-GPU: one process per GPU (torchrun), each rank an independent replica on
its own batch (the layer has no exchange step), so value = all tokens / max
rank time and scaling is weak.

Timing: per step, L2 is flushed (a 256 MiB write) outside the timed events,
then CUDA events on the launching stream bracket the forward; the timed region
is bracketed by a barrier and device synchronisation and the result is the
maximum over ranks.  Stage timing (CUDA events recorded by the library around
each kernel) gives the live duration of the dominant kernel for the roofline.
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


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="olmoe_like", choices=sorted(synth.WORKLOADS))
    p.add_argument("--tokens", type=int, default=32)
    p.add_argument("--numerics", default="exact", choices=["exact", "a4"])
    p.add_argument("--slots", default="workload", choices=["workload", "all"],
                   help="resident budget: the workload's own, or every expert resident")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU baseline sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay leg")
    return p.parse_args()


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
    block scales of every active expert, the f16 activations read once, and h written."""
    per_expert = 2 * wl.inter * wl.hidden * (0.5 + 1.0 / wl.group)
    return n_active * per_expert + T * wl.hidden * 2 + T * wl.top_k * wl.inter * 2


def layer_bytes(wl, n_active, T):
    """Algorithmic HBM bytes of one forward (unique active experts read once + router +
    shared expert + x + y)."""
    b = n_active * wl.expert_bytes() + wl.n_experts * wl.hidden * 4 + T * wl.hidden * (2 + 4)
    if wl.shared_inter:
        b += 3 * wl.shared_inter * wl.hidden * 2
    return b


def traffic_record(summary, kernel_src):
    """DRAM bytes per launch from a committed ncu summary (profiles/<summary>), if it
    was taken on the kernel source as it is now (its sha256 is recorded there)."""
    path = os.path.join(ROOT, "profiles", summary)
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

    _, r = layer.forward(x, routing=True)
    torch.cuda.synchronize()
    n_active = int((r["counts"] > 0).sum().item())

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
    # per-stage device times: a separate pass of the same loop with the
    # library's stage event pairs on, so that they do not touch the timed steps
    layer.profile_enable(True)
    for i in range(min(K, 200)):
        flush.zero_()
        layer.forward_ptr(x.data_ptr(), T, y.data_ptr(), sp)
    torch.cuda.synchronize()
    prof = layer.profile_read()
    layer.profile_enable(False)
    dev_ms = sum(a.elapsed_time(b) for a, b in zip(ev0, ev1))

    # e2e through the public host-buffer call: H2D of x, forward, D2H of y
    e2e = None
    if not args.no_e2e:
        xh = torch.from_numpy(x_bits.view(np.int16)).pin_memory()
        yh = torch.empty((T, wl.hidden), dtype=torch.float32).pin_memory()
        Ke = max(10, K // 4)
        for _ in range(5):
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

    vals = torch.tensor([dev_ms, e2e[0] if e2e else 0.0, graph_ms], dtype=torch.float64, device=dev)
    vals = max_over_ranks(vals, world)
    dev_ms_max, e2e_ms_max, graph_ms_max = float(vals[0]), float(vals[1]), float(vals[2])

    if rank == 0:
        hbm_peak, bf16_peak, bf16_sus, peak_src = peaks()
        ms_step = dev_ms_max / K
        value = whole_job_tokens_per_s(world, T, K, dev_ms_max)
        g_ms = prof["ms"]["gateup"] / max(1, prof["launches"]["gateup"])
        if args.numerics == "a4":
            # tcgen05 gate/up GEMM: FP4 FLOPs of the real (unpadded) token rows
            waves = max(1.0, prof["launches"]["gateup"] / max(1, prof["forwards"]))
            g_flops = 4.0 * T * wl.top_k * wl.hidden * wl.inter / waves
            achieved = g_flops / (g_ms / 1e3) / 1e12
            # the GEMM runs back to back for seconds inside the step loop: sustained figure
            fp4_peak = 4.0 * bf16_sus
            roof = {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                    "frac": achieved / fp4_peak, "traffic": None,
                    "kernel": "gemm_a4_kernel gate/up+SwiGLU (tcgen05 block-scaled FP4)",
                    "peak_source": f"{peak_src} bf16_tflops_sustained x 4 (nominal FP4/BF16 dense ratio)",
                    "algorithmic_flops_per_launch": g_flops, "kernel_ms": g_ms,
                    "hbm_gbs_of_same_launch": gateup_bytes(wl, n_active, T) / (g_ms / 1e3) / 1e9}
        else:
            # paged runs launch the pass once per staging wave: bytes per launch
            waves = max(1.0, prof["launches"]["gateup"] / max(1, prof["forwards"]))
            g_bytes = gateup_bytes(wl, n_active, T) / waves
            achieved = g_bytes / (g_ms / 1e3) / 1e9
            tc = wl.fmt == "mxfp4"
            src = os.path.join(ROOT, "fp4_expert_layer_b200", "csrc", "expert_tc.cu" if tc else "expert_tma.cu")
            traffic = None
            if tc and wl.name == "olmoe_like" and T == 32 and S == wl.n_experts:
                traffic = traffic_record("expert_tc_gateup_olmoe_like_T32.md", src)
            roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak, "traffic": traffic,
                    "kernel": ("expert_tc_kernel gate/up+SwiGLU (tcgen05, E2M1 weights x E4M3 activation pieces)"
                               if tc else "expert_tma_kernel gate/up+SwiGLU (register decode, mma.sync)"),
                    "peak_source": f"{peak_src} hbm_gbs",
                    "algorithmic_bytes_per_launch": g_bytes, "kernel_ms": g_ms}
        stage_ms = {k: v / max(1, prof["forwards"]) for k, v in prof["ms"].items()}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16xfp4->f32" if args.numerics == "exact" else "fp4xfp4->f32",
            "data": "synthetic (seeded; random-init weights of the workload's shape)",
            "config": {"workload": wl.name, "tokens": T, "hidden": wl.hidden, "inter": wl.inter,
                       "n_experts": wl.n_experts, "top_k": wl.top_k, "fmt": wl.fmt,
                       "shared_inter": wl.shared_inter, "resident_slots": S, "numerics": args.numerics,
                       "parallelism": f"replicas x{world}", "l2": "flushed (256 MiB write) before every step",
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
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(lw, x_bits, args.cpu_seconds, args.numerics)
        print(json.dumps(line), flush=True)

    layer.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
