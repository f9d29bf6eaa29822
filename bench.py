"""Benchmark of the ternary-weight MoE FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload: one decode-shape layer (d_model 2048, 256 experts, top-8, d_ff 512,
ternary 2-bit weights, seed 0) run on the four decode batches T = 1, 8, 32
and 64 (105 tokens).  A step is one forward pass of the whole layer (routing,
permutation, gate/up, down, combine) for each of the four batches.  Before
every forward pass L2 is flushed (a 256 MB write, outside the timed events),
so the weights come from HBM.  Each forward is a replay of a CUDA graph of the
library call (its two kernels), timed with CUDA events on its stream; the step
time is their sum.  value = tokens per second over all ranks.  The per-stage
split (routing / experts) comes from a second set of graphs that also record
the library's stage events, replayed after the timed region.

The JSON line adds: roofline (dominant kernel vs measured HBM bandwidth),
cpu_baseline (the CPU oracle timed on a sample), e2e (host buffers with the
copies inside the timed region), clocks sampled during the timed region, and
gpu_launches.

With N > 1 every rank runs its own replica on its own tokens (the layer
shards by tokens with no exchange): scaling is weak, timing is the max over
ranks.  --impl reference times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DECODE_T = (1, 8, 32, 64)
METRIC = "MoE-layer tokens/s (decode T=1..64, prefill T=4096) and % HBM/int8 roofline"
WORKLOAD = "decode-shape ternary MoE layer: d_model=2048, 256 experts, top-8, d_ff=512, T in {1,8,32,64}"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------- clocks
def pci_bus_id(dev) -> str | None:
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.proc = None
        self.bus_id = bus_id

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus_id:
            cmd += ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        pass

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- ranks
def reduce_max_over_ranks(values, device=None):
    """Max over ranks of per-rank device timings (identity on one process)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return units_per_rank * world / (max_ms * 1e-3)


# ---------------------------------------------------------------------------- measured traffic
PROFILE_T64 = os.path.join(ROOT, "profiles", "decode_experts_kernel__decode_T64.md")


def csrc_digest() -> str:
    """sha256 over the CUDA sources (file names and contents, sorted)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "ternary_weight_moe_forward_b200", "csrc", "*"))):
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic():
    """DRAM bytes (read + write) of one T=64 launch of decode_experts_kernel from
    the committed ncu summary, or None when the sources changed since."""
    try:
        with open(PROFILE_T64) as f:
            txt = f.read()
        fields = dict(line.split(": ", 1) for line in txt.splitlines()
                      if line.startswith(("csrc_sha256: ", "traffic_bytes: ")))
        if fields.get("csrc_sha256", "").strip() != csrc_digest():
            return None
        return int(fields["traffic_bytes"])
    except (OSError, KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------- GPU arm
def decode_bytes(n_active: int, T: int) -> int:
    """Algorithmic HBM bytes of one decode forward: packed codes and scales of
    the experts touched, the fp32 router matrix, x in (bf16) and y out (fp32)."""
    D, E, F = 2048, 256, 512
    per_expert = 3 * F * D // 4 + (2 * F + D) * 4
    return n_active * per_expert + E * D * 4 + T * D * 2 + T * D * 4


def experts_bytes(n_active: int, T: int) -> int:
    """Algorithmic bytes of the expert-stage kernel (decode_experts_kernel):
    packed codes and scales of the experts touched (gate, up, down), the int8
    activations in and the fp32 layer output."""
    D, F = 2048, 512
    return n_active * (3 * F * D // 4 + (2 * F + D) * 4) + T * D + T * D * 4


def run_gpu(args, rank: int, world: int):
    import torch
    import torch.distributed as dist

    import ternary_weight_moe_forward_b200 as tw
    from ternary_weight_moe_forward_b200 import synth
    from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    shape = synth.CONFIGS["decode"]["shape"]
    weights = synth.layer_weights(shape, seed=0)
    layer = Layer(shape, weights, max_tokens=max(DECODE_T), device=dev)
    del weights
    stream = torch.cuda.current_stream(dev)
    xs = {T: bf16_from_bits(synth.activations(T, shape.d_model, seed=0, stream=rank), dev) for T in DECODE_T}
    ys = {T: torch.empty((T, shape.d_model), dtype=torch.float32, device=dev) for T in DECODE_T}
    n_active = {}
    for T in DECODE_T:
        _, _, counts = layer.route(xs[T])
        n_active[T] = int((counts > 0).sum().item())
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    # One CUDA graph per batch size: the forward (routing kernel, permutation
    # and expert kernel) replays without host launch gaps.  The library's
    # per-stage events are captured with it, so the stages are timed on the
    # device as well.
    ev = {T: [torch.cuda.Event(enable_timing=True) for _ in range(4)] for T in DECODE_T}
    for T in DECODE_T:
        for e in ev[T]:
            e.record(stream)
    torch.cuda.synchronize(dev)
    # Two graphs per batch size: the timed one holds only the library's kernels;
    # the second also records the per-stage events (an event between the routing
    # and the expert kernel would keep them from overlapping their launch) and
    # gives the stage split after the timed region.
    graphs, split_graphs = {}, {}
    for T in DECODE_T:
        layer.forward(xs[T], y=ys[T])          # warm the path before capture
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer.forward(xs[T], y=ys[T])
        graphs[T] = g
        tw.maple_moe_set_stage_events(layer.handle, ev[T])
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer.forward(xs[T], y=ys[T])
        split_graphs[T] = g
        tw.maple_moe_set_stage_events(layer.handle, None)
    torch.cuda.synchronize(dev)

    e_beg = {T: torch.cuda.Event(enable_timing=True) for T in DECODE_T}
    e_end = {T: torch.cuda.Event(enable_timing=True) for T in DECODE_T}
    stages_in_graph = True

    def one_step(timed: list | None):
        for T in DECODE_T:
            flush.fill_(1.0)
            e_beg[T].record(stream)
            graphs[T].replay()
            e_end[T].record(stream)
            if timed is not None:
                torch.cuda.synchronize(dev)
                timed.append((T, e_beg[T].elapsed_time(e_end[T]), None))

    def split_step():
        """Stage times (route, gate/up, experts end) from the graphs with events."""
        nonlocal stages_in_graph
        out = {}
        for T in DECODE_T:
            flush.fill_(1.0)
            split_graphs[T].replay()
            torch.cuda.synchronize(dev)
            try:
                out[T] = [ev[T][0].elapsed_time(ev[T][i]) for i in range(1, 4)]
            except Exception:
                stages_in_graph = False
                return None
        return out

    for _ in range(args.warmup):
        one_step(None)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clk = ClockSampler(pci_bus_id(dev))
    clk.__enter__()
    timed = []
    for _ in range(args.steps):
        one_step(timed)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = clk.stop()

    # stage split: the same number of forwards again, from the graphs with events
    split = {T: [] for T in DECODE_T}
    for _ in range(args.steps):
        sp = split_step()
        if sp is None:
            break
        for T in DECODE_T:
            split[T].append(sp[T])
    if stages_in_graph:
        stage_src = "events inside a second set of graphs (untimed replays)"
        timed = [(T, tot, split[T][n % len(split[T])]) for n, (T, tot, _) in enumerate(timed)]

    if not stages_in_graph:
        # stage split from host-launched forwards instead (same kernels, stage events on the stream)
        stage_src = "host-launched forwards"
        split = {T: [] for T in DECODE_T}
        tw.maple_moe_set_stage_events(layer.handle, None)
        for _ in range(args.steps):
            for T in DECODE_T:
                flush.fill_(1.0)
                tw.maple_moe_set_stage_events(layer.handle, ev[T])
                layer.forward(xs[T], y=ys[T])
                torch.cuda.synchronize(dev)
                split[T].append([ev[T][0].elapsed_time(ev[T][i]) for i in range(1, 4)])
        tw.maple_moe_set_stage_events(layer.handle, None)
        timed = [(T, tot, split[T][n % len(split[T])]) for n, (T, tot, _) in enumerate(timed)]

    total_ms = sum(t[1] for t in timed)
    per_T = {T: [t[2] for t in timed if t[0] == T] for T in DECODE_T}
    fwd_T = {T: [t[1] for t in timed if t[0] == T] for T in DECODE_T}
    experts_ms = sum(x[2] - x[0] for T in DECODE_T for x in per_T[T])
    experts_alg = sum(experts_bytes(n_active[T], T) for T in DECODE_T) * args.steps

    # ---- end to end: pinned host x -> device, forward, y -> pinned host, all timed
    hx = {T: xs[T].cpu().pin_memory() for T in DECODE_T}
    hy = {T: torch.empty((T, shape.d_model), dtype=torch.float32).pin_memory() for T in DECODE_T}
    dx = {T: torch.empty_like(xs[T]) for T in DECODE_T}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for it in range(args.warmup + args.steps):
        for T in DECODE_T:
            flush.fill_(1.0)
            e0.record(stream)
            dx[T].copy_(hx[T], non_blocking=True)
            layer.forward(dx[T], y=ys[T])
            hy[T].copy_(ys[T], non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if it >= args.warmup:
                e2e_ms += e0.elapsed_time(e1)

    # ---- max over ranks
    total_ms, e2e_ms, experts_ms = reduce_max_over_ranks([total_ms, e2e_ms, experts_ms], device=dev)
    tokens_rank = sum(DECODE_T) * args.steps
    hbm, peak_kind = peaks()
    achieved = experts_alg / (experts_ms * 1e-3) / 1e9
    layer_bytes = sum(decode_bytes(n_active[T], T) for T in DECODE_T) * args.steps
    out = {
        "metric": METRIC,
        "value": whole_job_rate(tokens_rank, world, total_ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded ternary weights P=.3/.4/.3, lognormal alpha, N(0,1) bf16 x)",
        "config": {"workload": WORKLOAD, "tokens_per_step": sum(DECODE_T), "layers": 1,
                   "experts_touched": {str(T): n_active[T] for T in DECODE_T},
                   "l2": "flushed before every timed forward (256 MB write, outside the events)",
                   "parallelism": f"replicas x{world}"},
        "per_T": {str(T): {"tokens_per_s": T / (statistics.mean(fwd_T[T]) * 1e-3),
                           "us_per_forward": 1e3 * statistics.mean(fwd_T[T]),
                           "us_route": 1e3 * statistics.mean(x[0] for x in per_T[T]),
                           "us_experts": 1e3 * statistics.mean(x[2] - x[0] for x in per_T[T]),
                           "layer_hbm_frac": decode_bytes(n_active[T], T) /
                           (statistics.mean(fwd_T[T]) * 1e-3) / 1e9 / hbm}
                  for T in DECODE_T},
        "layer_roofline_frac": layer_bytes / (total_ms * 1e-3 / world) / 1e9 / hbm if world == 1 else None,
        "roofline": {"kernel": "decode_experts_kernel", "bound": "hbm", "achieved": achieved, "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": measured_traffic(), "traffic_launch": "T=64 (ncu, profiles/)",
                     "algorithmic_bytes_T64": experts_bytes(n_active[64], 64)},
        "e2e": {"value": whole_job_rate(tokens_rank, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(T * shape.d_model * 2 for T in DECODE_T),
                "d2h_bytes_per_step": sum(T * shape.d_model * 4 for T in DECODE_T)},
        "gpu_launches": 2 * len(DECODE_T) * args.steps,
        "cuda_graphs": True,
        "stage_split_from": stage_src,
        "clocks": clocks,
    }
    return out, layer


def cpu_baseline(seconds_cap: float = 20.0) -> dict:
    """Time the CPU oracle (single thread) on a sample of the same workload:
    up to 8 tokens of each decode batch (25 tokens), the router over all
    experts and the expert FFNs of every kept expert."""
    import oracle
    from ternary_weight_moe_forward_b200 import synth
    shape = synth.CONFIGS["decode"]["shape"]
    L = oracle.Layer(shape, synth.layer_weights(shape, seed=0))
    n_tok = 0
    t0 = time.perf_counter()
    for T in DECODE_T:
        x = synth.activations(T, shape.d_model, seed=0)
        n = min(T, 8)
        L.forward_tokens(x[:n], taps=False)
        n_tok += n
    dt = time.perf_counter() - t0
    return {"value": n_tok / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n_tok} tokens (first <=8 of each decode batch T=1,8,32,64), single-threaded C oracle, {dt:.1f} s"}


def run_reference(args):
    """The CPU oracle as the reference arm: each step = the 25-token sample."""
    import oracle
    from ternary_weight_moe_forward_b200 import synth
    shape = synth.CONFIGS["decode"]["shape"]
    L = oracle.Layer(shape, synth.layer_weights(shape, seed=0))
    xs = {T: synth.activations(T, shape.d_model, seed=0)[:min(T, 8)] for T in DECODE_T}
    per_step = sum(x.shape[0] for x in xs.values())
    for _ in range(args.warmup):
        for x in xs.values():
            L.forward_tokens(x, taps=False)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for x in xs.values():
            L.forward_tokens(x, taps=False)
    dt = time.perf_counter() - t0
    v = per_step * args.steps / dt
    sample = f"{per_step} tokens per step (first <=8 of each decode batch T=1,8,32,64), single-threaded C oracle"
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": {"workload": WORKLOAD},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    out, layer = run_gpu(args, rank, world)
    layer.close()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline()
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
