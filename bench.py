"""Benchmark of the ternary-weight MoE FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload: the decode-shape layer (d_model 2048, 256 experts, top-8, d_ff 512,
ternary 2-bit weights) run on the four decode batches T = 1, 8, 32 and 64 (105
tokens), each through 32 independently seeded layers (6.4 GB of packed
weights), one forward pass of the whole layer (routing, permutation, gate/up,
down, combine) per layer: a step is 4 x 32 layer forwards.  The inputs are
larger than L2: consecutive forwards read different layers' weights, as a
model's layers follow one another (at T = 1 the 32 layers touch about 270 MB,
twice the 126 MB L2).  Per batch size one CUDA graph holds the 32 forwards
(four kernels each); its replay is timed with CUDA events on the stream, and
the step time is the sum over the four batch sizes.  value = layer-tokens per
second (tokens x layers) over all ranks.  The per-stage split (routing /
gate-up / down + combine) comes from single-forward graphs that also record
the library's stage events, replayed once per layer after the timed region.
per_T also reports each batch with L2 flushed before every forward (a 256 MB
write, outside the events), which also evicts the kernels' instructions.

The JSON line adds: roofline (dominant kernel vs measured HBM bandwidth),
cpu_baseline (the CPU oracle timed on a sample, pinned to one host core),
e2e (host buffers with the copies inside the timed region), clocks sampled
during the timed region, gpu_launches, and per_config: the other workloads
of the layer, each timed the same way (CUDA graph replays, L2 flushed before
each, CUDA events on the stream): prefill T = 4096 (tensor-core path, with
its grouped GEMMs against the int8 tensor peak), the skewed-routing layer at
T = 16384, the 24-layer stack at T = 1 and 32, and the tiny layer.

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


def int8_peak_tops():
    """Dense int8 tensor peak, TOPS: the measured bf16 burst GEMM rate times the
    nominal int8 : bf16 ratio of the part (4.5 : 2.25 PFLOP/s = 2)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return 2.0 * float(p["bf16_tflops"]), "2 x measured bf16 burst (nominal int8:bf16 = 2)"
    except Exception:
        return 2.0 * 1590.0, "2 x fallback bf16 1590 TFLOP/s (nominal int8:bf16 = 2)"


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
PROFILE_T64 = os.path.join(ROOT, "profiles", "decode_stage_kernel__decode_T64.md")
# the sources of the dominant kernel (decode_stage_kernel): its own file and
# the helpers and layout it is built from
TRAFFIC_SOURCES = ("common.cuh", "decode.cuh", "layout.cuh")


def csrc_digest() -> str:
    """sha256 over the dominant kernel's CUDA sources (file names and contents,
    in TRAFFIC_SOURCES order; a missing file counts as empty)."""
    import hashlib
    h = hashlib.sha256()
    for name in TRAFFIC_SOURCES:
        h.update(name.encode())
        try:
            with open(os.path.join(ROOT, "ternary_weight_moe_forward_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        except OSError:
            pass
    return h.hexdigest()


def measured_traffic():
    """DRAM bytes (read + write) of one T=64 launch of decode_stage_kernel<1>
    from the committed ncu summary, or None when its sources changed since."""
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
    """Algorithmic bytes of the expert stage (gate/up, down and combine kernels):
    packed codes and scales of the experts touched (gate, up, down), the int8
    activations in and the fp32 layer output."""
    D, F = 2048, 512
    return n_active * (3 * F * D // 4 + (2 * F + D) * 4) + T * D + T * D * 4


def gate_up_bytes(n_active: int, T: int) -> int:
    """Algorithmic bytes of the gate/up kernel: gate and up codes and scales of
    the experts touched, the int8 activations in, h out (fp32, T*K rows)."""
    D, F, K = 2048, 512, 8
    return n_active * (2 * F * D // 4 + 2 * F * 4) + T * D + T * K * F * 4



def expected_experts(T: int, E: int = 256, K: int = 8) -> float:
    """Expected number of distinct experts a batch of T tokens touches under
    uniform routing."""
    return E * (1.0 - ((E - K) / E) ** T)


def prefill_ops(S: int, D: int = 2048, F: int = 512) -> tuple[int, int]:
    """int8 operations (2 per multiply-add) of the two grouped GEMMs for S slots."""
    return 2 * S * (2 * F) * D, 2 * S * D * F


class GraphTimer:
    """One library call captured as a CUDA graph (plus a second capture that
    also records the library's stage events), replayed after an L2 flush and
    timed with CUDA events on the stream."""

    def __init__(self, fn, stream, flush, set_events=None, n_events: int = 4):
        import torch
        self.torch, self.stream, self.flush = torch, stream, flush
        fn()
        torch.cuda.synchronize()
        # captured on torch's capture stream (fn reads torch's current stream),
        # replayed on `stream`
        self.g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g):
            fn()
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_events)]
        self.gs = None
        if set_events is not None:
            for e in self.ev:
                e.record(stream)
            torch.cuda.synchronize()
            set_events(self.ev)
            self.gs = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.gs):
                fn()
            set_events(None)
        self.e0 = torch.cuda.Event(enable_timing=True)
        self.e1 = torch.cuda.Event(enable_timing=True)

    def replay_ms(self) -> float:
        self.flush.fill_(1.0)
        self.e0.record(self.stream)
        self.g.replay()
        self.e1.record(self.stream)
        self.torch.cuda.synchronize()
        return self.e0.elapsed_time(self.e1)

    def stages_ms(self):
        """Stage boundaries (ms after the first event), from the graph with events."""
        if self.gs is None:
            return None
        self.flush.fill_(1.0)
        self.gs.replay()
        self.torch.cuda.synchronize()
        return [self.ev[0].elapsed_time(e) for e in self.ev[1:]]

    def run(self, steps: int, warmup: int):
        for _ in range(warmup):
            self.replay_ms()
        t = [self.replay_ms() for _ in range(steps)]
        st = [self.stages_ms() for _ in range(steps)] if self.gs is not None else None
        return t, st


def _mean_stage(st, i):
    return statistics.mean(x[i] - (x[i - 1] if i > 0 else 0.0) for x in st)


def bench_prefill(args, dev, stream, flush, hbm, name, T, zipf, seed_x):
    """One prefill-shape layer at T tokens on the tensor-core path."""
    import torch

    import ternary_weight_moe_forward_b200 as tw
    from ternary_weight_moe_forward_b200 import synth
    from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits
    shape = synth.CONFIGS["decode"]["shape"]
    w = synth.layer_weights_device(shape, seed=0, zipf=zipf, device=dev)
    layer = Layer(shape, w, max_tokens=T, device=dev)
    del w
    x = bf16_from_bits(synth.activations(T, shape.d_model, seed=seed_x), dev)
    y = torch.empty((T, shape.d_model), dtype=torch.float32, device=dev)
    _, _, counts = layer.route(x)
    counts = counts.cpu().numpy()
    gt = GraphTimer(lambda: layer.forward(x, y=y), stream, flush,
                    lambda ev: tw.maple_moe_set_stage_events(layer.handle, ev))
    t, st = gt.run(args.steps, args.warmup)
    fwd = statistics.mean(t)
    S = T * shape.top_k
    ops_gu, ops_dn = prefill_ops(S)
    peak, peak_kind = int8_peak_tops()
    us = {"route_and_permute": 1e3 * _mean_stage(st, 0), "gate_up_stage": 1e3 * _mean_stage(st, 1),
          "down_stage": 1e3 * _mean_stage(st, 2)}
    gemm_us = us["gate_up_stage"] + us["down_stage"]

    def roof(kernel, ops, u):
        a = ops / (u * 1e-6) / 1e12
        return {"kernel": kernel, "bound": "tensor", "dtype": "int8", "achieved": a, "peak": peak,
                "peak_kind": peak_kind, "unit": "TOPS", "frac": a / peak, "ops": ops}

    # end to end: pinned host x in, forward, y out, all inside the events
    hx = x.cpu().pin_memory()
    hy = torch.empty((T, shape.d_model), dtype=torch.float32).pin_memory()
    dx = torch.empty_like(x)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e = []
    for it in range(args.warmup + args.steps):
        flush.fill_(1.0)
        e0.record(stream)
        dx.copy_(hx, non_blocking=True)
        layer.forward(dx, y=y)
        hy.copy_(y, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            e2e.append(e0.elapsed_time(e1))
    layer.close()
    out = {
        "workload": f"{name}: d_model=2048, 256 experts, top-8, d_ff=512, T={T}"
                    + (", Zipf(1.1) router bias" if zipf else ""),
        "tokens_per_s": T / (fwd * 1e-3), "us_per_forward": 1e3 * fwd, "us_stages": us,
        "experts_touched": int((counts > 0).sum()), "max_tokens_per_expert": int(counts.max()),
        "roofline_gemms": roof("gate/up + down stages (grouped GEMMs with their epilogue kernels)",
                               ops_gu + ops_dn, gemm_us),
        "roofline_gate_up": roof("gate/up stage", ops_gu, us["gate_up_stage"]),
        "roofline_down": roof("down stage (incl. combine)", ops_dn, us["down_stage"]),
        "e2e": {"value": T / (statistics.mean(e2e) * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * shape.d_model * 2, "d2h_bytes_per_step": T * shape.d_model * 4},
    }
    return out


def bench_stack(args, dev, stream, flush, hbm):
    """The 24-layer stack (RMSNorm + layer, residual) at T = 1 and 32, one graph."""
    import torch

    import ternary_weight_moe_forward_b200 as tw
    from ternary_weight_moe_forward_b200 import synth
    from ternary_weight_moe_forward_b200.layer import Layer
    cfg = synth.CONFIGS["stack"]
    shape = cfg["shape"]
    layers = []
    for l in range(cfg["layers"]):
        w = synth.layer_weights_device(shape, seed=1000, layer=l, device=dev)
        layers.append(Layer(shape, w, max_tokens=max(cfg["tokens"]), device=dev, flags=tw.MAPLE_CFG_DECODE_ONLY))
        del w
    torch.cuda.synchronize()
    handles = [L.handle for L in layers]
    out = {}
    for T in cfg["tokens"]:
        r0 = torch.from_numpy(synth.residual(T, shape.d_model, seed=T)).to(dev)
        resid = r0.clone()

        def step():
            resid.copy_(r0)
            tw.maple_moe_stack_forward(handles, resid, T, torch.cuda.current_stream(dev).cuda_stream)

        gt = GraphTimer(step, stream, flush)
        t, _ = gt.run(args.steps, args.warmup)
        ms = statistics.mean(t)
        n_exp = expected_experts(T)
        byts = cfg["layers"] * decode_bytes(int(round(n_exp)), T)
        out[str(T)] = {"tokens_per_s": T / (ms * 1e-3), "us_per_step": 1e3 * ms,
                       "hbm_frac": byts / (ms * 1e-3) / 1e9 / hbm,
                       "bytes_note": f"expected distinct experts per layer {n_exp:.1f} (uniform routing)"}
    for L in layers:
        L.close()
    return {"workload": "24-layer MoE-FFN stack (pre-norm RMSNorm + residual), d_model=2048, 256 experts, "
                        "top-8, d_ff=512, independent layers", "per_T": out}


def bench_tiny(args, dev, stream, flush):
    import torch

    from ternary_weight_moe_forward_b200 import synth
    from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits
    shape = synth.CONFIGS["tiny"]["shape"]
    layer = Layer(shape, synth.layer_weights(shape, seed=0), max_tokens=8, device=dev)
    x = bf16_from_bits(synth.activations(8, shape.d_model, seed=0), dev)
    y = torch.empty((8, shape.d_model), dtype=torch.float32, device=dev)
    gt = GraphTimer(lambda: layer.forward(x, y=y), stream, flush)
    t, _ = gt.run(args.steps, args.warmup)
    layer.close()
    return {"workload": "tiny: d_model=256, 16 experts, top-2, d_ff=128, T=8", "us_per_forward": 1e3 * statistics.mean(t),
            "tokens_per_s": 8 / (statistics.mean(t) * 1e-3), "bound": "latency"}


N_ROT = 32   # layers in rotation: their weights (6.4 GB) are the inputs larger than L2


def run_gpu(args, rank: int, world: int):
    import torch
    import torch.distributed as dist

    import ternary_weight_moe_forward_b200 as tw
    from ternary_weight_moe_forward_b200 import synth
    from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    shape = synth.CONFIGS["decode"]["shape"]
    layers = []
    for l in range(N_ROT):
        w = synth.layer_weights_device(shape, seed=0, layer=l, device=dev)
        layers.append(Layer(shape, w, max_tokens=max(DECODE_T), device=dev, flags=tw.MAPLE_CFG_DECODE_ONLY))
        del w
    stream = torch.cuda.current_stream(dev)
    xs = {T: bf16_from_bits(synth.activations(T, shape.d_model, seed=0, stream=rank), dev) for T in DECODE_T}
    ys = {T: torch.empty((T, shape.d_model), dtype=torch.float32, device=dev) for T in DECODE_T}
    # the expert path of each batch size (the library decides: the fused kernel
    # where all of a batch's expert clusters fit on the device at once)
    fused = {T: tw.maple_moe_expert_path(layers[0].handle, T) == tw.MAPLE_PATH_DECODE_FUSED for T in DECODE_T}
    n_active = {T: [] for T in DECODE_T}   # experts touched, per layer
    for T in DECODE_T:
        for L in layers:
            _, _, counts = L.route(xs[T])
            n_active[T].append(int((counts > 0).sum().item()))
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    no_flush = torch.empty(0, dtype=torch.float32, device=dev)

    # The timed unit: per batch size one CUDA graph holding the forwards of all
    # N_ROT layers in order (each forward is two or four kernels, each a programmatic
    # dependent of the one before); one replay = N_ROT forwards, back to back,
    # timed with CUDA events on the stream.  Consecutive forwards read different
    # layers' weights.
    seq = {T: GraphTimer(lambda T=T: [L.forward(xs[T], y=ys[T]) for L in layers], stream, no_flush)
           for T in DECODE_T}
    # one forward per graph, with the library's stage events (an event between two
    # kernels keeps them from overlapping their launch): the stage split, replayed
    # once per layer after the timed region
    single = {(T, l): GraphTimer(lambda T=T, L=L: L.forward(xs[T], y=ys[T]), stream, no_flush,
                                 lambda ev, L=L: tw.maple_moe_set_stage_events(L.handle, ev))
              for T in DECODE_T for l, L in enumerate(layers)}

    def one_step(timed: list | None):
        for T in DECODE_T:
            ms = seq[T].replay_ms()
            if timed is not None:
                timed.append((T, ms))

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

    # stage split: every layer once more, from the graphs with events
    split = {T: [(l, single[(T, l)].stages_ms()) for l in range(N_ROT)] for T in DECODE_T}
    stage_src = "events inside single-forward graphs (untimed replays, every layer once)"
    # the same batches with L2 flushed before each forward (layer 0): code and data cold
    flushed = {T: [] for T in DECODE_T}
    for T in DECODE_T:
        gt = single[(T, 0)]
        gt.flush = flush
        for _ in range(args.warmup):
            gt.replay_ms()
        flushed[T] = [gt.replay_ms() for _ in range(args.steps)]
        gt.flush = no_flush

    total_ms = sum(t[1] for t in timed)
    fwd_T = {T: [t[1] / N_ROT for t in timed if t[0] == T] for T in DECODE_T}
    experts_ms = sum(x[2] - x[0] for T in DECODE_T for _, x in split[T])
    experts_alg = sum(experts_bytes(n_active[T][l], T) for T in DECODE_T for l, _ in split[T])
    # the gate/up kernel of the two-kernel path (the batches that take it)
    gu_ms = sum(x[1] - x[0] for T in DECODE_T if not fused[T] for _, x in split[T])
    gu_alg = sum(gate_up_bytes(n_active[T][l], T) for T in DECODE_T if not fused[T] for l, _ in split[T])

    # ---- end to end: pinned host x -> device, forward, y -> pinned host, all timed
    hx = {T: xs[T].cpu().pin_memory() for T in DECODE_T}
    hy = {T: torch.empty((T, shape.d_model), dtype=torch.float32).pin_memory() for T in DECODE_T}
    dx = {T: torch.empty_like(xs[T]) for T in DECODE_T}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for it in range(args.warmup + args.steps):
        for T in DECODE_T:
            e0.record(stream)
            dx[T].copy_(hx[T], non_blocking=True)
            for L in layers:
                L.forward(dx[T], y=ys[T])
            hy[T].copy_(ys[T], non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if it >= args.warmup:
                e2e_ms += e0.elapsed_time(e1)
    del seq, single
    for L in layers:
        L.close()
    del layers
    torch.cuda.empty_cache()

    # ---- max over ranks
    total_ms, e2e_ms, experts_ms = reduce_max_over_ranks([total_ms, e2e_ms, experts_ms], device=dev)
    tokens_rank = sum(DECODE_T) * N_ROT * args.steps   # each step: the four batches through every layer
    hbm, peak_kind = peaks()
    achieved = experts_alg / (experts_ms * 1e-3) / 1e9
    layer_bytes = sum(decode_bytes(n_active[T][l], T) for T in DECODE_T for l in range(N_ROT)) * args.steps
    gu_achieved = gu_alg / (gu_ms * 1e-3) / 1e9
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
        "config": config_of(world),
        "experts_touched_mean": {str(T): statistics.mean(n_active[T]) for T in DECODE_T},
        "l2": f"inputs larger than L2: {N_ROT} independently seeded layers (6.4 GB of packed weights) "
              "in rotation, one per forward; no flush inside the timed region",
        "per_T": {str(T): per_T_entry(T, fused[T], fwd_T[T], flushed[T], split[T], n_active[T], hbm) for T in DECODE_T},
        "layer_roofline_frac": layer_bytes / (total_ms * 1e-3 / world) / 1e9 / hbm if world == 1 else None,
        "roofline": {"kernel": "decode_stage_kernel<1> (gate/up: the dominant kernel; batches of 32 and 64)",
                     "bound": "hbm",
                     "achieved": gu_achieved, "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": gu_achieved / hbm, "traffic": measured_traffic(),
                     "traffic_launch": "T=64 (ncu, profiles/)",
                     "algorithmic_bytes_T64": gate_up_bytes(round(statistics.mean(n_active[64])), 64)},
        "roofline_expert_stage": {"kernels": "dx_fused_kernel (T in " + str([T for T in DECODE_T if fused[T]]) +
                                             "); decode_stage_kernel<1>, decode_stage_kernel<2>, dx_combine_kernel "
                                             "(the others)",
                                  "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                                  "frac": achieved / hbm},
        "e2e": {"value": whole_job_rate(tokens_rank, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(T * shape.d_model * 2 for T in DECODE_T),
                "d2h_bytes_per_step": sum(T * shape.d_model * 4 for T in DECODE_T)},
        # per forward: routing + the fused expert kernel (T <= 8), or routing, gate/up, down, combine
        "gpu_launches": sum(2 if fused[T] else 4 for T in DECODE_T) * N_ROT * args.steps,
        "cuda_graphs": True,
        "stage_split_from": stage_src,
        "clocks": clocks,
    }
    if not args.decode_only:
        # the other workloads, each on its own (timed after the headline's region)
        per = {}
        per["prefill"] = bench_prefill(args, dev, stream, flush, hbm, "prefill", 4096, None, 0)
        per["skewed"] = bench_prefill(args, dev, stream, flush, hbm, "skewed routing", 16384, 1.1, 5)
        per["stack"] = bench_stack(args, dev, stream, flush, hbm)
        per["tiny"] = bench_tiny(args, dev, stream, flush)
        out["per_config"] = per
        out["roofline_prefill"] = per["prefill"]["roofline_gemms"]
    return out


def per_T_entry(T, fused, fwd, flushed, split, n_active, hbm) -> dict:
    """One decode batch size's line: times per forward and the stage split
    (routing; experts: gate/up and down + combine, or the fused expert kernel)."""
    ent = {"tokens_per_s": T / (statistics.mean(fwd) * 1e-3),
           "us_per_forward": 1e3 * statistics.mean(fwd),
           "us_per_forward_l2_flushed": 1e3 * statistics.mean(flushed),
           "expert_path": "fused" if fused else "two-kernel",
           "us_route": 1e3 * statistics.mean(x[0] for _, x in split),
           "us_experts": 1e3 * statistics.mean(x[2] - x[0] for _, x in split),
           "layer_hbm_frac": statistics.mean(decode_bytes(n, T) for n in n_active) /
           (statistics.mean(fwd) * 1e-3) / 1e9 / hbm,
           "experts_hbm_frac": statistics.mean(experts_bytes(n_active[l], T) / ((x[2] - x[0]) * 1e-3) / 1e9 / hbm
                                               for l, x in split)}
    if not fused:
        ent["us_gate_up"] = 1e3 * statistics.mean(x[1] - x[0] for _, x in split)
        ent["us_down_combine"] = 1e3 * statistics.mean(x[2] - x[1] for _, x in split)
        ent["gate_up_hbm_frac"] = statistics.mean(gate_up_bytes(n_active[l], T) / ((x[1] - x[0]) * 1e-3) / 1e9 / hbm
                                                  for l, x in split)
    return ent


def config_of(world: int) -> dict:
    return {"workload": WORKLOAD, "layers": N_ROT, "layer_tokens_per_step": sum(DECODE_T) * N_ROT,
            "parallelism": f"replicas x{world}"}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class pinned_to_one_core:
    """Run the enclosed block on a single host core (the first one this
    process may use); restores the affinity afterwards."""

    def __enter__(self):
        self.old = os.sched_getaffinity(0)
        self.core = min(self.old)
        os.sched_setaffinity(0, {self.core})
        return self

    def __exit__(self, *a):
        os.sched_setaffinity(0, self.old)


def _oracle_sample():
    """The oracle's sample of the workload: the first <= 8 tokens of each decode
    batch (T = 1, 8, 32, 64: 25 tokens) and 16 tokens of the T = 4096 prefill
    batch, all through the full layer (router over every expert, the kept
    experts' FFNs, combine)."""
    from ternary_weight_moe_forward_b200 import synth
    shape = synth.CONFIGS["decode"]["shape"]
    xs = [synth.activations(T, shape.d_model, seed=0)[:min(T, 8)] for T in DECODE_T]
    xs.append(synth.activations(4096, shape.d_model, seed=0)[:16])
    return shape, xs


def cpu_baseline() -> dict:
    """Time the CPU oracle, single-threaded and pinned to one core, on its sample."""
    import oracle
    from ternary_weight_moe_forward_b200 import synth
    shape, xs = _oracle_sample()
    L = oracle.Layer(shape, synth.layer_weights(shape, seed=0))
    n_tok = sum(x.shape[0] for x in xs)
    with pinned_to_one_core() as pin:
        t0 = time.perf_counter()
        for x in xs:
            L.forward_tokens(x, taps=False)
        dt = time.perf_counter() - t0
    return {"value": n_tok / dt, "unit": "tokens/s", "cores": 1, "cores_total": os.cpu_count(),
            "cpu_model": cpu_model(), "pinned_core": pin.core, "kind": "oracle",
            "sample": f"{n_tok} tokens: first <=8 of each decode batch T=1,8,32,64 and 16 of the T=4096 prefill "
                      f"batch; single-threaded C oracle on 1 of {os.cpu_count()} cores, {dt:.1f} s"}


def run_reference(args):
    """The CPU oracle as the reference arm: each step = the oracle's sample
    (tokens are independent, so its tokens/s is that of the whole workload)."""
    import oracle
    from ternary_weight_moe_forward_b200 import synth
    shape, xs = _oracle_sample()
    L = oracle.Layer(shape, synth.layer_weights(shape, seed=0))
    per_step = sum(x.shape[0] for x in xs)
    with pinned_to_one_core() as pin:
        for _ in range(args.warmup):
            for x in xs:
                L.forward_tokens(x, taps=False)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            for x in xs:
                L.forward_tokens(x, taps=False)
        dt = time.perf_counter() - t0
    v = per_step * args.steps / dt
    sample = (f"{per_step} tokens per step (first <=8 of each decode batch T=1,8,32,64 and 16 of the T=4096 "
              f"prefill batch), single-threaded C oracle on 1 of {os.cpu_count()} cores")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": config_of(1),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "cores_total": os.cpu_count(),
                             "cpu_model": cpu_model(), "pinned_core": pin.core, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-only", action="store_true", help="skip the per_config workloads")
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
    out = run_gpu(args, rank, world)
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
