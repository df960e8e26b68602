#!/usr/bin/env python
"""Benchmark of the CQS-decomposed exact attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 oracle on host cores

One step = one pass of the whole path over the workload's synthetic input.
The default workload is CQS l=4 (13 chunks of 4096), N=53248, H=8, d=128,
bf16, device-resident, run non-causal and causal: a step is both forwards.
Metric: useful TFLOP/s, 4 N^2 H d per forward (halved when causal).

Rank 0 prints one JSON line.  Under torchrun every rank runs its own
independent problem (weak scaling, no collective on the data path); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GiB = 1 << 30
L2_BYTES = 126 * 1000 * 1000

# name -> workload.  "variants" are the causal settings one step runs.
WORKLOADS = {
    "cqs-l4-n53248-h8-d128-bf16-device": dict(
        N=53248, H=8, d=128, ls=[4], dtype="bf16", mode="device", variants=[False, True],
        dist="normal", budget=0),
    "cqs-l3-n3584-h1-d64-fp32-device": dict(
        N=3584, H=1, d=64, ls=[3], dtype="fp32", mode="device", variants=[False],
        dist="normal", budget=0),
    "cqs-l5-n688128-h8-d128-bf16-host-2gib": dict(
        N=688128, H=8, d=128, ls=[5], dtype="bf16", mode="host", variants=[False],
        dist="normal", budget=2 * GiB),
    "cqs-l4l3-n1490944-h4-d128-bf16-host-4gib-causal": dict(
        N=1490944, H=4, d=128, ls=[4, 3], dtype="bf16", mode="host", variants=[True],
        dist="normal", budget=4 * GiB),
    "cqs-l6-n2031616-h1-d128-bf16-host-2gib": dict(
        N=2031616, H=1, d=128, ls=[6], dtype="bf16", mode="host", variants=[False],
        dist="half_normal_uniform_v", budget=2 * GiB),
}
DEFAULT_WORKLOAD = "cqs-l4-n53248-h8-d128-bf16-device"
# Extra keys of the default one-GPU line: one host-streamed workload and the
# fp32 workload, each measured the same way as its own --workload line.
STREAMED_EXTRA = "cqs-l6-n2031616-h1-d128-bf16-host-2gib"
FP32_EXTRA = "cqs-l3-n3584-h1-d64-fp32-device"
METRIC = "exact-attention TFLOP/s (4*N^2*H*d, halved for causal)"


# ------------------------------------------------------------------ helpers
def useful_flops(N: int, H: int, d: int, causal: bool) -> float:
    return 4.0 * N * N * H * d * (0.5 if causal else 1.0)


def merge_bytes(plan, info, ebytes: int) -> float:
    """HBM bytes the slots merge must move for one forward: every partial of
    every query block read once (O_j fp32 and lse_j), out and lse written."""
    N, H, d, blk = info["N"], info["H"], info["d"], info["block_tokens"]
    parts = 0
    for i in range(info["num_entries"]):
        b = plan.entry(i)["q_block"]
        parts += max(0, min((b + 1) * blk, N) - b * blk)
    return float(parts) * H * (4 * d + 4) + float(N) * H * (ebytes * d + 4)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def profile_traffic(kernel_file: str, summary: str):
    """Per-launch DRAM bytes recorded in a committed ncu summary, or None when
    the kernel source has changed since the counters were taken."""
    try:
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        src = open(os.path.join(ROOT, "out_core_scheduling_b200", "csrc", kernel_file), "rb").read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_source_sha256") != hashlib.sha256(src).hexdigest():
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock, power and throttle reasons with nvidia-smi."""

    QUERY = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.device_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, parts[3:]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for_smi(torch, dev: int) -> str:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x for x in vis.split(",") if x.strip()]
        return ids[dev] if dev < len(ids) else str(dev)


# ------------------------------------------------------------------ distributed
class Dist:
    """Rank bookkeeping; torch.distributed only when launched by torchrun."""

    def __init__(self, backend: str | None = None):
        import torch.distributed as dist
        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.on = self.world > 1
        if self.on and not dist.is_initialized():
            import datetime
            dist.init_process_group(backend=backend or "nccl",
                                    timeout=datetime.timedelta(seconds=120))

    def barrier(self, device=None):
        if self.on:
            if device is not None and self.dist.get_backend() == "nccl":
                self.dist.barrier(device_ids=[device])
            else:
                self.dist.barrier()

    def max(self, x: float, device="cpu") -> float:
        if not self.on:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.on and self.dist.is_initialized():
            self.dist.destroy_process_group()


# ------------------------------------------------------------ sharded arm
def run_sharded(args, W, D=None, workload=None):
    """--shard: ONE problem of the workload split over the ranks (strong
    scaling): every rank plans with shard_rank = its rank, computes its
    (task, query block) entries with cqsa_forward_partial, and the ranks
    exchange their log-sum-exp partials over NCCL: an all-to-all to each
    query block's owner, the owner's merge, an all-gather of the merged rows
    (out_core_scheduling_b200.sharded).  Launched without torchrun it runs
    on a one-process NCCL group.  Device workloads only.

    Given D (the default run's ranks, N > 1), it returns the line as a dict
    and leaves the process group open; otherwise rank 0 prints it."""
    import datetime
    import socket

    import torch
    import torch.distributed as dist
    from out_core_scheduling_b200 import cqsa
    from out_core_scheduling_b200.inputs import make_qkv
    from out_core_scheduling_b200.sharded import forward_sharded

    if W["mode"] != "device":
        raise SystemExit("--shard takes a device workload")
    nested = D is not None
    workload = workload or args.workload
    D = D or Dist()
    dev = D.local_rank
    torch.cuda.set_device(dev)
    torch_dev = f"cuda:{dev}"
    cqsa.load_library()
    if not dist.is_initialized():
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(port))
        dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(torch_dev))
    rank, world = dist.get_rank(), dist.get_world_size()
    N, H, d = W["N"], W["H"], W["d"]
    tdt = torch.bfloat16 if W["dtype"] == "bf16" else torch.float32
    cdt = cqsa.CQSA_BF16 if W["dtype"] == "bf16" else cqsa.CQSA_FP32
    q, k, v = make_qkv(N, H, d, dtype=tdt, seed=0, device=torch_dev, dist=W["dist"])  # the same problem everywhere
    plans = [cqsa.cqsa_plan_ex(N, H, d, W["ls"], causal=c, dtype=cdt, shard_rank=rank, shard_count=world)
             for c in W["variants"]]
    outs = [torch.empty_like(q) for _ in plans]
    lses = [torch.empty(H, N, device=torch_dev) for _ in plans]
    flops_step = sum(useful_flops(N, H, d, c) for c in W["variants"])

    def step():
        for p, o, l in zip(plans, outs, lses):
            forward_sharded(p, q, k, v, o, l)

    for _ in range(args.warmup):
        step()
    for p in plans:
        p.sync()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(gpu_id_for_smi(torch, dev))
    for p in plans:
        p.kernel_stats(reset=True)
        p.profile(True)
    sampler.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier(dev)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    D.barrier(dev)
    clocks = sampler.stop()
    for p in plans:
        p.profile(False)
        p.sync()
    stats = [p.kernel_stats(reset=True) for p in plans]
    ms = D.max(ev0.elapsed_time(ev1), torch_dev)
    value = flops_step * args.steps / (ms * 1e-3) / 1e12
    infos = [p.info() for p in plans]
    from out_core_scheduling_b200.sharded import exchange_bytes
    exch = sum(exchange_bytes(p) for p in plans)
    exch_ar = sum(exchange_bytes(p, "allreduce") for p in plans)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": W["dtype"], "data": "synthetic (seeded torch.Generator, see inputs.py)",
        "config": {"workload": workload, "N": N, "H": H, "d": d, "l": W["ls"], "causal": W["variants"],
                   "mode": "device, task shards", "parallelism": f"one problem in {world} task shards",
                   "l2": "inputs larger than L2; no flush"},
        "shard": {"rank0_entries": [i["shard_entries"] for i in infos],
                  "rank0_pair_share": [i["shard_pairs"] / i["total_pairs"] for i in infos],
                  "exchange": "owners: all-to-all of partials to each query block's owner, owner-side "
                              "log-sum-exp merge, all-gather of the merged rows",
                  "exchange_bytes_per_rank_per_step": exch,
                  "exchange_bytes_two_all_reduces": exch_ar,
                  "collectives_per_step": 2 * len(plans)},
        "clocks": clocks,
        # attention (none on a rank without entries) + partial init + owner merge
        "gpu_launches": sum(s["attn_launches"] for s in stats) + 2 * len(plans) * args.steps,
    }
    for p in plans:
        p.destroy()
    if nested:
        return line
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()


# ------------------------------------------------------------------ our arm
def run_ours(args, W):
    """The default line: the workload's step, and with the default workload
    on one GPU also the streamed l=6 workload and the fp32 workload as extra
    keys ("streamed", "fp32_small"); with N > 1 GPUs the task-sharded step
    of the same problem as the extra key "sharded"."""
    import torch
    from out_core_scheduling_b200 import cqsa

    D = Dist()
    torch.cuda.set_device(D.local_rank)
    cqsa.load_library()  # fails loudly when the library is missing
    result = measure(args, W, D, args.workload, args.steps, args.warmup, extras=True)
    if result is None:  # --profile-run
        D.close()
        return
    if args.workload == DEFAULT_WORKLOAD and not args.no_extra:
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        if D.world == 1:
            sub = argparse.Namespace(**vars(args))
            sub.no_e2e = sub.no_cpu = True
            if sub.backward_host_steps < 0:
                sub.backward_host_steps = 1
            result["streamed"] = measure(sub, WORKLOADS[STREAMED_EXTRA], D, STREAMED_EXTRA,
                                         args.streamed_steps, 3, extras=False)
            torch.cuda.empty_cache()
            result["fp32_small"] = measure(sub, WORKLOADS[FP32_EXTRA], D, FP32_EXTRA,
                                           args.steps, max(3, args.warmup), extras=False)
        else:
            result["sharded"] = run_sharded(args, W, D=D, workload=args.workload)
    if D.rank == 0:
        print(json.dumps(result), flush=True)
    D.close()


def flush_l2(buf):
    """Overwrite a buffer larger than L2, so the next launch starts cold."""
    buf.add_(1)


def measure(args, W, D, workload, steps, warmup, extras):
    """One workload's line (a dict) on this rank's GPU; every rank runs its
    own independent problem and the step time is the max over ranks."""
    import torch
    from out_core_scheduling_b200 import cqsa
    from out_core_scheduling_b200.inputs import make_qkv

    dev = D.local_rank
    torch_dev = f"cuda:{dev}"
    N, H, d = W["N"], W["H"], W["d"]
    tdt = torch.bfloat16 if W["dtype"] == "bf16" else torch.float32
    cdt = cqsa.CQSA_BF16 if W["dtype"] == "bf16" else cqsa.CQSA_FP32
    ebytes = 2 if W["dtype"] == "bf16" else 4
    seed = D.rank  # each rank: its own independent problem

    plans = [cqsa.cqsa_plan_ex(N, H, d, W["ls"], causal=c, dtype=cdt, mem_budget_bytes=W["budget"])
             for c in W["variants"]]
    infos = [p.info() for p in plans]
    flops_step = sum(useful_flops(N, H, d, c) for c in W["variants"])
    stream = torch.cuda.current_stream()

    free_before, _ = torch.cuda.mem_get_info()
    if W["mode"] == "device":
        q, k, v = make_qkv(N, H, d, dtype=tdt, seed=seed, device=torch_dev, dist=W["dist"])
        outs = [torch.empty_like(q) for _ in plans]
        lses = [torch.empty(H, N, device=torch_dev, dtype=torch.float32) for _ in plans]
        mode = cqsa.CQSA_DEVICE
        io_bytes = (3 + len(plans)) * q.numel() * ebytes + sum(x.numel() * 4 for x in lses)
    else:
        gq, gk, gv = make_qkv(N, H, d, dtype=tdt, seed=seed, device=torch_dev, dist=W["dist"])
        q, k, v = (x.cpu().pin_memory() for x in (gq, gk, gv))
        del gq, gk, gv
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        free_before, _ = torch.cuda.mem_get_info()
        outs = [torch.empty(q.shape, dtype=tdt).pin_memory() for _ in plans]
        lses = [torch.empty(H, N, dtype=torch.float32).pin_memory() for _ in plans]
        mode = cqsa.CQSA_HOST
        io_bytes = 0

    def step():
        for p, o, l in zip(plans, outs, lses):
            cqsa.cqsa_forward(p, q, k, v, o, l, mode, stream)

    for _ in range(warmup):
        step()
    for p in plans:
        p.sync(stream)
    free_after, _ = torch.cuda.mem_get_info()

    if args.profile_run:
        for _ in range(steps):
            step()
        if args.profile_backward and mode == cqsa.CQSA_DEVICE:
            dout = make_qkv(N, H, d, dtype=tdt, seed=1000 + D.rank, device=q.device, dist=W["dist"])[0]
            grads = tuple(torch.empty_like(q) for _ in range(3))
            for _ in range(steps):  # first variant only: one backward arena on the device
                cqsa.cqsa_backward(plans[0], q, k, v, outs[0], lses[0], dout, *grads, stream=stream)
        for p in plans:
            p.sync(stream)
        return None

    # Inputs smaller than L2 (the fp32 workload): each timed step starts after
    # a write of a buffer larger than L2, outside the events that time it.
    in_bytes = 3 * N * H * d * ebytes
    flush = (torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=torch_dev).zero_()
             if mode == cqsa.CQSA_DEVICE and in_bytes <= L2_BYTES else None)

    sampler = ClockSampler(gpu_id_for_smi(torch, dev))
    for p in plans:
        p.kernel_stats(reset=True)
        p.profile(True)
    sampler.start()
    time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps if flush is not None else 1)]
    D.barrier(dev)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    if flush is None:
        evs[0][0].record(stream)
        for _ in range(steps):
            step()
        evs[0][1].record(stream)
    else:
        for e0, e1 in evs:
            flush_l2(flush)
            e0.record(stream)
            step()
            e1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    D.barrier(dev)
    clocks = sampler.stop()
    for p in plans:
        p.profile(False)
        p.sync(stream)
    ms = D.max(sum(e0.elapsed_time(e1) for e0, e1 in evs), torch_dev)
    stats = [p.kernel_stats(reset=True) for p in plans]

    value = flops_step * steps * D.world / (ms * 1e-3) / 1e12
    peaks = load_peaks()

    # Roofline of the dominant kernel: the tile-attention launch of the first
    # variant (non-causal for the default workload), its useful flops over
    # its mean event-timed duration on the stream it was launched on.
    attn_ms = sum(s["attn_ms"] for s in stats)
    attn_launches = sum(s["attn_launches"] for s in stats)
    s0 = stats[0]
    launch_ms = s0["attn_ms"] / max(1, s0["attn_launches"])
    flops_per_forward = useful_flops(N, H, d, W["variants"][0])
    if W["mode"] == "device":
        achieved = flops_per_forward / (launch_ms * 1e-3) / 1e12 if launch_ms > 0 else None
    else:  # one launch per task: all the forward's flops over all its launches
        achieved = flops_per_forward * steps / (s0["attn_ms"] * 1e-3) / 1e12 if s0["attn_ms"] else None
    if W["dtype"] == "bf16":
        # A device-mode launch is timed alone (burst peak); a streamed step
        # runs the tensor cores for seconds (sustained peak).
        sustained = W["mode"] != "device"
        peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak if achieved else None,
                    "peak_source": peaks["source"] + (" bf16 dense (sustained)" if sustained
                                                      else " bf16 dense (burst)"),
                    "traffic": (profile_traffic("attn_tc.cu", "attn_tc_l4_n53248_h8_d128.md")
                                if workload == DEFAULT_WORKLOAD else None),
                    "kernel": f"attn_tc_kernel<{d}> (causal={W['variants'][0]})",
                    "avg_launch_ms": launch_ms}
    else:
        # fp32 FFMA on the CUDA cores: 148 SMs x 128 FMA/clk x 2 flops x max clock.
        peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roofline = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak if achieved else None,
                    "peak_source": "fp32 FFMA: 148 SMs x 128 lanes x 2 x 1965 MHz",
                    "traffic": (profile_traffic("attn_simt.cu", "attn_simt_l3_n3584_h1_d64_fp32.md")
                                if workload == FP32_EXTRA else None),
                    "kernel": f"attn_simt_kernel<{d}>",
                    "avg_launch_ms": launch_ms}
    merge = None
    merge_ms = sum(s["merge_ms"] for s in stats)
    merge_launches = sum(s["merge_launches"] for s in stats)
    if W["mode"] == "device" and merge_ms > 0:
        mb = 0.0
        for p, info, s in zip(plans, infos, stats):
            mb += merge_bytes(p, info, ebytes) * s["merge_launches"]
        merge = {"bound": "hbm", "achieved": mb / (merge_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                 "unit": "GB/s", "frac": mb / (merge_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                 "bytes_per_launch": mb / max(1, merge_launches), "kernel": "merge_slots_kernel",
                 "note": "algorithmic bytes: each query block's partials (4d+4 B per row and head each, "
                         "as many as the block has entries) read once, the output and lse written once"}

    arena = sum(i["device_arena_bytes"] if W["mode"] == "device" else i["host_arena_bytes"] for i in infos)
    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": D.world,
        "steps": steps, "warmup": warmup, "ms_per_step": ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": W["dtype"], "data": "synthetic (seeded torch.Generator, see inputs.py)",
        "config": {"workload": workload, "N": N, "H": H, "d": d, "l": W["ls"],
                   "c": [info["c"] for info in infos[:1]][0], "D": infos[0]["D"],
                   "causal": W["variants"], "mode": W["mode"],
                   "mem_budget_bytes": W["budget"] or None,
                   "parallelism": f"independent problem per GPU x{D.world}",
                   "l2": (f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB > 126 MB); no flush" if flush is None
                          else f"inputs {in_bytes / 1e6:.1f} MB < L2: a {flush.numel() * 4 / 1e6:.0f} MB buffer "
                               "is written before every timed step, outside its events")},
        "roofline": roofline,
        "roofline_merge": merge,
        "clocks": clocks,
        "gpu_launches": attn_launches + merge_launches,
        "per_variant": [{"causal": c, "tflops_kernel": useful_flops(N, H, d, c) * steps
                         / (s["attn_ms"] * 1e-3) / 1e12 if s["attn_ms"] else None,
                         "attn_ms_per_launch": s["attn_ms"] / max(1, s["attn_launches"]),
                         "merge_ms_per_launch": s["merge_ms"] / max(1, s["merge_launches"])}
                        for c, s in zip(W["variants"], stats)],
        "peak_hbm_gib": {"library_arena": arena / GiB, "inputs_outputs": io_bytes / GiB,
                         "device_free_delta": (free_before - free_after) / GiB},
        "wall_ms_timed": (wall1 - wall0) * 1e3,
    }

    # ---- the fused recomposition on the same device inputs (no slots, no
    # merge launch), timed the same way; the headline stays the slots path.
    if W["mode"] == "device" and extras and not args.no_fused:
        result["fused_merge"] = run_fused(args, W, D, q, k, v, outs, lses, flops_step, stream, value)
    # ---- the backward of the same problems (device mode).
    if W["mode"] == "device" and extras and not args.no_backward:
        result["backward"] = run_backward(args, W, D, plans, q, k, v, outs, lses, flops_step, stream, peaks)

    # ---- end to end through the public API from pinned host memory.
    if W["mode"] == "host":
        # The timed path already starts and ends in pinned host memory.
        h2d = int(sum(i["h2d_bytes"] for i in infos))
        d2h = int(sum(i["d2h_bytes"] for i in infos))
        result["e2e"] = {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                         "d2h_bytes_per_step": d2h, "ms_per_step": ms / steps,
                         "path": "cqsa_forward(CQSA_HOST), the timed path itself"}
        result["streaming"] = streaming_report(W, infos, flops_step, ms / steps, peaks,
                                               free_before, torch)
        if args.backward_host_steps > 0:
            result["backward_streamed"] = run_backward_host(args, W, D, plans, infos, q, k, v, outs, lses,
                                                            flops_step, stream, peaks, result["streaming"])
    elif not args.no_e2e:
        result["e2e"] = run_e2e(args, W, D, plans, infos, q, k, v, flops_step, stream, extras)

    # ---- oracle on the host cores (rank 0, N = 1 only).
    if D.rank == 0 and D.world == 1 and not args.no_cpu:
        # About 10-20 s of fp64 work on the host cores, whatever the workload.
        rows = args.cpu_rows or max(8, min(512, int(2.5e11 / (W["H"] * W["N"] * 4 * W["d"]))))
        result["cpu_baseline"] = cpu_baseline(W, q, k, v, rows)

    for p in plans:
        p.destroy()
    return result


def run_backward(args, W, D, plans, q, k, v, outs, lses, flops_step, stream, peaks):
    """cqsa_backward after each variant's forward outputs, with a seeded
    output gradient; useful flops 2.5x the forward's (S, dP, dQ, dK, dV
    against S, PV)."""
    import torch
    from out_core_scheduling_b200 import cqsa
    from out_core_scheduling_b200.inputs import make_qkv

    N, H, d = W["N"], W["H"], W["d"]
    tdt = q.dtype
    dout = make_qkv(N, H, d, dtype=tdt, seed=1000 + D.rank, device=q.device, dist=W["dist"])[0]
    grads = [tuple(torch.empty_like(q) for _ in range(3)) for _ in plans]

    def step():
        for p, o, l, g in zip(plans, outs, lses, grads):
            cqsa.cqsa_backward(p, q, k, v, o, l, dout, *g, stream=stream)

    for p, o, l in zip(plans, outs, lses):
        cqsa.cqsa_forward(p, q, k, v, o, l, cqsa.CQSA_DEVICE, stream)
    for _ in range(args.warmup):
        step()
    for p in plans:
        p.sync(stream)
        p.kernel_stats(reset=True)
        p.profile(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier(D.local_rank)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    D.barrier(D.local_rank)
    for p in plans:
        p.profile(False)
        p.sync(stream)
    stats = [p.kernel_stats(reset=True) for p in plans]
    ms = D.max(ev0.elapsed_time(ev1), f"cuda:{D.local_rank}")
    bflops = 2.5 * flops_step
    value = bflops * args.steps * D.world / (ms * 1e-3) / 1e12
    bwd_ms = sum(s["bwd_ms"] for s in stats)
    kern = bflops * args.steps / (bwd_ms * 1e-3) / 1e12 if bwd_ms else None
    peak = peaks["bf16_tflops"] if W["dtype"] == "bf16" else 148 * 128 * 2 * 1.965e9 / 1e12
    return {"value": value, "unit": "TFLOP/s", "ms_per_step": ms / args.steps,
            "useful_flops_per_step": bflops,
            "gradient_kernels_tflops": kern, "frac_of_peak": kern / peak if kern else None,
            "peak": peak, "gpu_launches": sum(s["bwd_launches"] + s["merge_launches"] for s in stats),
            "path": "cqsa_backward: D = rowsum(dout * out); dq kernel over the (task, query block) list, "
                    "dk/dv kernel over the (task, key block) list, slot sums"}


def run_backward_host(args, W, D, plans, infos, q, k, v, outs, lses, flops_step, stream, peaks, fwd_stream):
    """cqsa_backward(CQSA_HOST) of each variant from pinned host memory under
    the workload's budget (the forward's outputs and a seeded pinned dout):
    2.5x the forward's useful flops per step, the bound from the sustained
    bf16 peak and the measured host link, and the device memory it takes."""
    import torch
    from out_core_scheduling_b200 import cqsa
    from out_core_scheduling_b200.inputs import make_qkv

    N, H, d = W["N"], W["H"], W["d"]
    gd = make_qkv(N, H, d, dtype=q.dtype, seed=1000 + D.rank, device=f"cuda:{D.local_rank}", dist=W["dist"])[0]
    dout = gd.cpu().pin_memory()
    del gd
    grads = [tuple(torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(3)) for _ in plans]
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    def step():
        for p, o, l, g in zip(plans, outs, lses, grads):
            cqsa.cqsa_backward(p, q, k, v, o, l, dout, *g, host_or_device=cqsa.CQSA_HOST, stream=stream)

    free0, _ = torch.cuda.mem_get_info()
    for _ in range(args.backward_host_warmup):
        step()
    for p in plans:
        p.sync(stream)
    free1, _ = torch.cuda.mem_get_info()
    sampler = ClockSampler(gpu_id_for_smi(torch, D.local_rank))
    sampler.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier(D.local_rank)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.backward_host_steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    D.barrier(D.local_rank)
    clocks = sampler.stop()
    for p in plans:
        p.sync(stream)
    ms = D.max(ev0.elapsed_time(ev1), f"cuda:{D.local_rank}") / args.backward_host_steps
    bflops = 2.5 * flops_step
    h2d = sum(i["bwd_h2d_bytes"] for i in infos)
    d2h = sum(i["bwd_d2h_bytes"] for i in infos)
    t_c = bflops / (peaks["bf16_tflops_sustained"] * 1e12) * 1e3
    t_h = h2d / (fwd_stream["h2d_gbs"] * 1e9) * 1e3
    t_d = d2h / (fwd_stream["d2h_gbs"] * 1e9) * 1e3
    bound = max(t_c, t_h, t_d)
    return {"value": bflops * D.world / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "steps": args.backward_host_steps, "warmup": args.backward_host_warmup,
            "useful_flops_per_step": bflops, "h2d_bytes": h2d, "d2h_bytes": d2h,
            "t_compute_at_peak_ms": t_c, "t_h2d_ms": t_h, "t_d2h_ms": t_d, "t_bound_ms": bound,
            "bound": "compute" if bound == t_c else ("h2d" if bound == t_h else "d2h"),
            "efficiency": bound / ms, "peak_source": "sustained bf16 dense",
            "head_group": infos[0]["bwd_head_group"], "cache_slots": infos[0]["bwd_cache_slots"],
            "num_blocks": infos[0]["num_blocks"], "writebacks_per_head_group": infos[0]["bwd_writebacks"],
            "library_arena_gib": max(i["bwd_host_arena_bytes"] for i in infos) / GiB,
            "device_free_delta_gib": (free0 - free1) / GiB, "budget_gib": W["budget"] / GiB,
            "clocks": clocks,
            "path": "cqsa_backward(CQSA_HOST): per head group lse up, D = rowsum(dout * out) per block, then "
                    "the leaf tasks through the backward block cache, gradient sums written back when evicted"}


def run_fused(args, W, D, q, k, v, outs, lses, flops_step, stream, slots_value):
    import torch
    from out_core_scheduling_b200 import cqsa

    N, H, d = W["N"], W["H"], W["d"]
    cdt = cqsa.CQSA_BF16 if W["dtype"] == "bf16" else cqsa.CQSA_FP32
    plans = [cqsa.cqsa_plan_ex(N, H, d, W["ls"], causal=c, dtype=cdt, merge=cqsa.CQSA_MERGE_FUSED)
             for c in W["variants"]]

    def step():
        for p, o, l in zip(plans, outs, lses):
            cqsa.cqsa_forward(p, q, k, v, o, l, cqsa.CQSA_DEVICE, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier(D.local_rank)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    D.barrier(D.local_rank)
    for p in plans:
        p.sync(stream)
    ms = D.max(ev0.elapsed_time(ev1), f"cuda:{D.local_rank}")
    value = flops_step * args.steps * D.world / (ms * 1e-3) / 1e12
    return {"value": value, "unit": "TFLOP/s", "ms_per_step": ms / args.steps,
            "vs_slots": value / slots_value if slots_value else None,
            "gpu_launches": len(plans) * args.steps,
            "path": "cqsa_plan_ex(merge=CQSA_MERGE_FUSED): one CTA per 256 query rows walks the allowed "
                    "key runs of all the tasks of its rows and writes out and lse; no slots, no merge launch"}


def run_e2e(args, W, D, plans, infos, q, k, v, flops_step, stream, extras=True):
    """The step through cqsa_forward(CQSA_HOST) from pinned host inputs to
    pinned host outputs.  The plans fit every block, so the resident
    schedule runs.  The step's problems are independent, so each goes on a
    stream of its own (joined at the end of every step) and one problem's
    copies overlap the other's kernels; the same calls on one stream, each
    problem alone, the task-by-task schedule (extras) and the device-resident
    step on the same streams are timed beside it."""
    import torch
    from out_core_scheduling_b200 import cqsa

    N, H = W["N"], W["H"]
    if W["mode"] == "host":
        hq, hk, hv = q, k, v
    else:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    outs = [torch.empty(hq.shape, dtype=hq.dtype).pin_memory() for _ in plans]
    lses = [torch.empty(H, N, dtype=torch.float32).pin_memory() for _ in plans]
    side = [torch.cuda.Stream() for _ in plans[1:]]

    def timed(ps, concurrent, host=True):
        ss = [stream] + side[:len(ps) - 1] if concurrent else [stream] * len(ps)
        fork = torch.cuda.Event()
        joins = [torch.cuda.Event() for _ in ps]
        if host:
            src, dst = (hq, hk, hv), list(zip(outs, lses))
            mode = cqsa.CQSA_HOST
        else:
            src = (q, k, v)
            dst = [(torch.empty_like(q), torch.empty(H, N, dtype=torch.float32, device=q.device)) for _ in ps]
            mode = cqsa.CQSA_DEVICE

        def step():
            if concurrent:
                fork.record(stream)
                for s in ss[1:]:
                    s.wait_event(fork)
            for p, (o, l), s in zip(ps, dst, ss):
                cqsa.cqsa_forward(p, *src, o, l, mode, s)
            if concurrent:
                for s, e in zip(ss[1:], joins[1:]):
                    e.record(s)
                    stream.wait_event(e)

        for _ in range(max(1, min(args.warmup, 3))):
            step()
        torch.cuda.synchronize()
        steps = max(1, min(args.steps, args.e2e_steps))
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        D.barrier(D.local_rank)
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        D.barrier(D.local_rank)
        for p, s in zip(ps, ss):
            p.sync(s)
        ms = D.max(ev0.elapsed_time(ev1), f"cuda:{D.local_rank}")
        return steps, ms

    def tflops(steps, ms, flops=flops_step):
        return flops * steps * D.world / (ms * 1e-3) / 1e12

    steps, ms = timed(plans, concurrent=len(plans) > 1)
    hinfo = [p.info() for p in plans]
    res = {"value": tflops(steps, ms), "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(sum(i["h2d_bytes"] for i in hinfo)),
           "d2h_bytes_per_step": int(sum(i["d2h_bytes"] for i in hinfo)),
           "steps": steps, "ms_per_step": ms / steps,
           "schedule": "resident" if all(i["host_resident"] for i in hinfo) else "tasks",
           "streams": len(plans),
           "path": "cqsa_forward(CQSA_HOST): pinned host q,k,v -> device block pools -> pinned host out,lse; "
                   "the step's independent problems on a stream each, joined every step"}
    if extras and len(plans) > 1:
        steps_1, ms_1 = timed(plans, concurrent=False)
        res["one_stream"] = {"value": tflops(steps_1, ms_1), "ms_per_step": ms_1 / steps_1,
                             "per_problem_ms": [ms_p / steps_p for steps_p, ms_p in (timed([p], False) for p in plans)]}
        steps_d, ms_d = timed(plans, concurrent=True, host=False)
        res["device_same_streams"] = {"value": tflops(steps_d, ms_d), "ms_per_step": ms_d / steps_d,
                                      "path": "cqsa_forward(CQSA_DEVICE) on the same streams: "
                                              "the device-resident step these copies are measured against"}
    if extras and res["schedule"] == "resident":
        tp = [cqsa.cqsa_plan_ex(N, H, W["d"], W["ls"], causal=i["causal"], dtype=i["dtype"], host_tasks=True)
              for i in hinfo]
        steps_t, ms_t = timed(tp, concurrent=False)
        res["tasks_schedule"] = {"value": tflops(steps_t, ms_t), "ms_per_step": ms_t / steps_t,
                                 "path": "the same calls on one stream, task by task "
                                         "(cqsa_plan_ex(host_tasks=True))"}
        for p in tp:
            p.destroy()
    return res


def host_link_gbs(torch, nbytes=1 << 30):
    """Pinned host <-> device copy bandwidth (GB/s), 1 GiB each way, best of 3."""
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = {}
    for name, dst, src in (("h2d", d, h), ("d2h", h, d)):
        best = None
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            dst.copy_(src, non_blocking=True)
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1)
            best = t if best is None else min(best, t)
        out[name] = nbytes / (best * 1e-3) / 1e9
    del h, d
    torch.cuda.empty_cache()
    return out


def streaming_report(W, infos, flops_step, ms_step, peaks, free_before, torch):
    """Streamed workloads: time bound = the slowest of compute at the bf16
    peak and each direction of the host link at its measured bandwidth;
    efficiency = bound / measured time; device memory against the budget.
    A streamed step keeps the tensor cores busy for seconds, so the compute
    bound uses the sustained peak; the burst-peak figure is reported beside
    it."""
    free_after, _ = torch.cuda.mem_get_info()
    link = host_link_gbs(torch)
    h2d = sum(i["h2d_bytes"] for i in infos)
    d2h = sum(i["d2h_bytes"] for i in infos)
    t_compute = flops_step / (peaks["bf16_tflops_sustained"] * 1e12) * 1e3
    t_compute_burst = flops_step / (peaks["bf16_tflops"] * 1e12) * 1e3
    t_h2d = h2d / (link["h2d"] * 1e9) * 1e3
    t_d2h = d2h / (link["d2h"] * 1e9) * 1e3
    bound = max(t_compute, t_h2d, t_d2h)
    which = ("compute" if bound == t_compute else "h2d" if bound == t_h2d else "d2h")
    min_in = 3 * W["N"] * W["H"] * W["d"] * 2
    return {"h2d_gbs": link["h2d"], "d2h_gbs": link["d2h"], "h2d_bytes": h2d, "d2h_bytes": d2h,
            "h2d_bytes_minimum": min_in, "t_compute_at_peak_ms": t_compute, "t_h2d_ms": t_h2d,
            "t_d2h_ms": t_d2h, "t_bound_ms": bound, "bound": which, "t_wall_ms": ms_step,
            "efficiency": bound / ms_step, "peak_tflops": peaks["bf16_tflops_sustained"],
            "peak_source": "sustained bf16 dense",
            "efficiency_at_burst_peak": max(t_compute_burst, t_h2d, t_d2h) / ms_step,
            "budget_gib": W["budget"] / GiB,
            "library_arena_gib": max(i["host_arena_bytes"] for i in infos) / GiB,
            "device_free_delta_gib": (free_before - free_after) / GiB,
            "head_group": infos[0]["head_group"], "tasks": infos[0]["num_tasks"]}


def oracle_sample(W, q, k, v, rows_per_variant, seed):
    """Time the fp64 oracle on a row sample of each variant; returns
    (useful flops of the sample, seconds, threads, description)."""
    import numpy as np
    import torch
    import oracle
    from out_core_scheduling_b200.inputs import sample_rows

    N, H, d = W["N"], W["H"], W["d"]
    qc, kc, vc = (x.cpu() if x.is_cuda else x for x in (q, k, v))
    flops, secs = 0.0, 0.0
    for i, causal in enumerate(W["variants"]):
        rows = sample_rows(N, rows_per_variant, seed=seed + i).numpy()
        keys = (rows + 1).sum() if causal else rows.size * N
        t0 = time.perf_counter()
        oracle.attention_rows(qc, kc, vc, rows=rows, causal=causal)
        secs += time.perf_counter() - t0
        flops += 4.0 * d * H * float(keys)
    desc = (f"{rows_per_variant} seeded query rows x {H} heads per variant "
            f"(causal={W['variants']}) against all allowed keys of the workload")
    return flops, secs, oracle.num_threads(), desc


def cpu_baseline(W, q, k, v, rows):
    flops, secs, threads, desc = oracle_sample(W, q, k, v, rows, seed=1234)
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": desc, "seconds": secs}


# ------------------------------------------------------------------ reference arm
def run_reference(args, W):
    """The fp64 oracle, as it stands, on the host cores: each step a bounded
    row sample of the workload.  Rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    from out_core_scheduling_b200.inputs import make_qkv

    tdt = torch.bfloat16 if W["dtype"] == "bf16" else torch.float32
    q, k, v = make_qkv(W["N"], W["H"], W["d"], dtype=tdt, seed=0, device="cpu", dist=W["dist"])
    for i in range(args.warmup):
        oracle_sample(W, q, k, v, args.ref_rows, seed=100 + i)
    flops, secs, threads, desc = 0.0, 0.0, 1, ""
    for i in range(args.steps):
        f, s, threads, desc = oracle_sample(W, q, k, v, args.ref_rows, seed=1000 + i)
        flops += f
        secs += s
    value = flops / secs / 1e12
    world = int(os.environ.get("WORLD_SIZE", "1"))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded torch.Generator, see inputs.py)",
        "config": {"workload": args.workload, "N": W["N"], "H": W["H"], "d": W["d"],
                   "l": W["ls"], "causal": W["variants"], "mode": "host cores (oracle)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="oracle rows per variant for cpu_baseline (0: sized to about 15 s)")
    ap.add_argument("--ref-rows", type=int, default=16, help="oracle rows per variant per reference step")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-fused", action="store_true", help="skip the fused-merge timing of device workloads")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing of device workloads")
    ap.add_argument("--profile-run", action="store_true",
                    help="only warm-up + steps of the device path (for ncu captures)")
    ap.add_argument("--profile-backward", action="store_true",
                    help="with --profile-run: the first variant's backward after the forward steps")
    ap.add_argument("--no-extra", action="store_true",
                    help="default workload: skip the streamed / fp32 (one GPU) or sharded (N > 1) extra keys")
    ap.add_argument("--streamed-steps", type=int, default=2,
                    help="timed steps of the streamed extra workload (about 2 s each)")
    ap.add_argument("--backward-host-steps", type=int, default=-1,
                    help="host-streamed workloads: timed steps of the host-mode backward "
                         "(default: 1 in the default run's streamed extra, 0 otherwise)")
    ap.add_argument("--backward-host-warmup", type=int, default=1)
    ap.add_argument("--shard", action="store_true",
                    help="one problem split over the ranks in task shards (strong scaling; not the default line)")
    args = ap.parse_args(argv)
    if args.warmup < 0 or args.steps < 1:
        ap.error("need --steps >= 1 and --warmup >= 0")
    W = WORKLOADS[args.workload]
    if args.backward_host_steps < 0 and not (args.workload == DEFAULT_WORKLOAD and not args.no_extra):
        args.backward_host_steps = 0
    if args.impl == "reference":
        run_reference(args, W)
    elif args.shard:
        run_sharded(args, W)
    else:
        run_ours(args, W)


if __name__ == "__main__":
    main()
