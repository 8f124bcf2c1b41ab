#!/usr/bin/env python3
"""Throughput of the grouped NVFP4 MoE expert forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--shared]
                    [--impl ours|reference]

One step = one layer forward: route sort, gate+up SiLU, down, blend (the four
C-ABI calls) over one batch of the workload's synthetic tokens, weights and
inputs resident in HBM.  The default workload is prefill M=8192, the largest
single-GPU one; ``--config`` picks another.  ``--shared`` adds the workload's
shared expert, run by every token inside the same launches (one more routing
slot).  The weights rotate over R device replicas (R x the routed bytes of a
step >= 4 x L2), so every step streams its expert weights from HBM.  The timed
region is one replay of a CUDA graph holding exactly ``--steps`` forwards,
bracketed by CUDA events on the launching stream (the median of per-replay
times of single-step graphs is reported beside it); under torchrun (N > 1)
each rank runs an independent replica of the workload (weak scaling, no
collective on the data path) and the time is the max over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
on the host cores instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 MoE layer tokens/s and routed-weight HBM GB/s (% of peak), 1 B200"
DEFAULT_CONFIG = "prefill_m8192"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# Default timed steps per workload: a fraction of a second to a second of GPU
# time each (all of them are captured in one CUDA graph).
DEFAULT_STEPS = {"tiny": 4000, "decode_m1": 4000, "decode_m32": 2000, "decode_m256": 300,
                 "prefill_m8192": 200}

# Sources of each projection kernel; their hash names the build an ncu capture
# was taken from.
KERNEL_SOURCES = {
    "tcgen05": ["grouped_tc.cu", "grouped_tc_pair.cuh", "tc_common.cuh", "common.cuh"],
    "mma.sync": ["grouped_mma.cu", "common.cuh"],
    "check_scales": ["check_scales.cu"],
    "transpose_u8": ["transpose_u8.cu"],
}

# DRAM bytes (read + write) of one launch of the dominant kernel (gate+up
# SiLU) from an ncu capture (summaries under profiles/), keyed by workload and
# kernel, with the hash of that kernel's sources when it was captured.  An
# entry whose hash no longer matches the sources is stale and not reported.
NCU_TRAFFIC_BYTES = {
    ("decode_m1", "mma.sync"): (28362496, "75ef290dff45"),       # 28.36 MB read, 0.002 MB written
    ("decode_m32", "tcgen05"): (297321728, "f284aa1030ca"),      # 293.13 MB read, 4.19 MB written
    # reduced case (64 experts, 64 tokens: the same 8 rows per expert) x 4 experts
    ("decode_m256", "tcgen05"): (4515166208, "f284aa1030ca"),    # 4 x (1122.08 + 6.71) MB
    ("prefill_m8192", "tcgen05"): (3189124864, "f284aa1030ca"),  # 2.7995 GB read, 0.3896 GB written
}
# Entries not captured on the workload itself: how the figure was obtained.
NCU_TRAFFIC_SCALED = {
    ("decode_m256", "tcgen05"): "4 x one launch of a 64-expert, 64-token case of the same "
                                "per-expert shape (the full workload is too large to capture)",
}


# The same for one launch of a load-time op's kernel (per projection for the
# scale check; per transposed matrix for the twins), keyed by op and workload.
NCU_OP_TRAFFIC_BYTES = {
    ("check_scales", "prefill_m8192"): (50353152, "5b4491c5e4d3"),   # 50.34 MB read, 0.01 MB written
    ("twins", "prefill_m8192"): (3150336, "07ac2b2c0b60"),           # packed part of one expert: 3.15 MB read
}


def kernel_source_hash(kernel: str) -> str:
    """First 12 hex digits of the SHA-256 over a projection kernel's sources."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "nvfp4_weight_quantized_moe_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def ncu_traffic(workload: str, kernel: str):
    """Captured DRAM bytes per launch, or None when absent or taken from other sources."""
    entry = NCU_TRAFFIC_BYTES.get((workload, kernel))
    if entry is None or entry[1] != kernel_source_hash(kernel):
        return None
    return entry[0]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["layer", "check_scales", "shard", "twins"], default="layer",
                    help="layer: the forward; check_scales / shard / twins: the load-time scale "
                         "check, tensor-parallel shard (--tp ranks, rank 0), or concatenated "
                         "gate|up transposed twin of every expert of the workload")
    ap.add_argument("--tp", type=int, default=2, help="tensor-parallel ranks for --op shard")
    ap.add_argument("--shared", action="store_true",
                    help="add a shared expert (every token, same launches as the routed experts)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--path", type=int, default=0, help="0 auto, 1 decode, 2 prefill")
    ap.add_argument("--split", type=int, default=0)
    ap.add_argument("--tiles", type=int, default=0)
    ap.add_argument("--depth", type=int, default=0)
    ap.add_argument("--staging", type=int, default=0,
                    help="decode path: 1 whole-K activation staging, 2 two-chunk ring, 0 auto")
    ap.add_argument("--no-workspace", action="store_true",
                    help="use the calls without workspace (decode path only)")
    ap.add_argument("--replicas", type=int, default=0,
                    help="weight replicas to rotate over (0: enough to exceed 4 x L2)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the workload's expert count (a reduced case for profiling)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (a reduced case for profiling)")
    return ap.parse_args(argv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def dist_info():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, group=None) -> float:
    """Max of a float over the ranks of the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# --------------------------------------------------------------------------- #
# Clock sampling during the timed region
# --------------------------------------------------------------------------- #

class ClockSampler:
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            rows.append((ts, parts))
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.06 <= r[0] <= self.t1 + 0.06]
        use = inside or rows[-3:]
        if not use:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[2]) for _, p in use if num(p[2]) is not None]
        smax = [num(p[3]) for _, p in use if num(p[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, p in use for i in range(4) if p[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(use), "samples_in_timed_region": len(inside)}


# --------------------------------------------------------------------------- #
# Our implementation
# --------------------------------------------------------------------------- #

def _replicate(layer, copies):
    """`copies` extra device copies of a layer's weights (distinct memory, same values)."""
    import nvfp4_weight_quantized_moe_b200 as nvm

    def clone(p):
        return nvm.NVFP4Projection(p.packed.clone(), p.scale.clone(), p.scale2.clone())

    out = [layer]
    for _ in range(copies):
        projs = [clone(p) for p in (layer.gate, layer.up, layer.down)]
        shared = tuple(clone(p) for p in layer.shared) if layer.shared is not None else None
        out.append(nvm.NVFP4MoE(*projs, layer.topk, shared=shared, shared_rows=layer.shared_rows))
    return out


def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    import nvfp4_weight_quantized_moe_b200 as nvm
    from workloads import make_problem
    from workloads.device import upload_inputs, upload_layer

    prob = make_problem(args.config, **_overrides(args))
    cfg = prob.cfg
    steps = args.steps if args.steps is not None else DEFAULT_STEPS.get(cfg.name, 1000)
    warmup = max(args.warmup, 3)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)

    base = upload_layer(prob, dev, shared=args.shared)
    x, ids, w = upload_inputs(prob, dev)
    bufs = base.buffers(cfg.tokens)
    ws = None if args.no_workspace else base.workspace(cfg.tokens)
    # Active experts of this batch (identical for every replica: same routing).
    with torch.cuda.stream(stream):
        base.forward(x, ids, w, bufs, workspace=ws, **_opts(args))
    stream.synchronize()
    if nvm.device_error() != 0:
        raise RuntimeError("device error word set by the forward")
    # With a shared expert, the forward runs topk + 1 slots over num_experts +
    # slots table entries; the shared expert's weights count once in the bytes.
    slots = 0
    topk_run, experts_run, pairs_run = cfg.topk, cfg.experts, cfg.pairs
    if args.shared:
        rows = base.rows_per_shared_slot(cfg.tokens)
        slots = nvm.shared_slots(cfg.tokens, rows)
        topk_run, experts_run = cfg.topk + 1, cfg.experts + slots
        pairs_run = cfg.tokens * topk_run
    active_all = int(bufs.active_count.item())
    active = active_all - slots
    per_expert = base.gate.nbytes_per_expert
    routed_bytes = 3 * (active + (1 if args.shared else 0)) * per_expert
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    replicas = max(1, math.ceil(4 * l2 / max(routed_bytes, 1)))
    free = torch.cuda.mem_get_info(dev)[0]
    layer_bytes = 3 * cfg.experts * per_expert
    replicas = int(min(replicas, max(1, (free * 0.6) // layer_bytes), 64))
    if args.replicas > 0:
        replicas = args.replicas
    layers = _replicate(base, replicas - 1)

    def step(lay):
        lay.forward(x, ids, w, bufs, workspace=ws, **_opts(args))

    # The timed region is ONE replay of a graph holding exactly `steps` layer
    # forwards, step i on replica i % R; nothing else is launched inside it.
    with torch.cuda.stream(stream):
        for lay in layers:
            step(lay)
    stream.synchronize()
    g_steps = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps, stream=stream):
        for i in range(steps):
            step(layers[i % len(layers)])
    # Single-step graphs, one per replica: warm-up and the per-replay median.
    g_one = []
    for lay in layers:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(lay)
        g_one.append(g)

    with torch.cuda.stream(stream):
        for i in range(warmup):
            g_one[i % len(layers)].replay()
        g_steps.replay()  # first replay of the big graph (uploads it), untimed
    stream.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.mark(True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        g_steps.replay()
        ev1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark(False)
    barrier()
    clocks = sampler.stop()
    elapsed_ms = reduce_max(ev0.elapsed_time(ev1))
    ms_per_step = elapsed_ms / steps
    tokens_per_s = world * cfg.tokens * steps / (elapsed_ms / 1e3)

    # Median over per-replay event times of single-step graphs (each replay
    # bracketed by its own events; replicas in turn), after the timed region.
    n_med = max(5, min(steps, 200))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_med)]
    with torch.cuda.stream(stream):
        for i, (a, b) in enumerate(evs):
            a.record(stream)
            g_one[i % len(layers)].replay()
            b.record(stream)
    torch.cuda.synchronize(dev)
    median_ms = reduce_max(statistics.median(a.elapsed_time(b) for a, b in evs))

    hbm, tflops, tflops_sus, peak_kind = measured_peaks()
    routed_gbs = world * routed_bytes / (ms_per_step * 1e-3) / 1e9

    # Dominant kernel, timed alone: gate+up SiLU, one launch per replica.
    tc = ws is not None and _tc_path(args, cfg, pairs_run, experts_run)
    prefill = tc and _uses_prefill(args, pairs_run, experts_run)
    gu_graph = torch.cuda.CUDAGraph()
    cap = nvm.active_cap(experts_run, pairs_run)

    def gate_up(lay):
        g, u = lay.gate.tables, lay.up.tables
        if args.shared:
            g, u = (t.tables for t in lay._ext_tables(slots)[:2])
        if ws is None:
            nvm.gate_up_silu(x, g, u, bufs.act, bufs.expert_offsets,
                             bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count,
                             cfg.inter, cfg.hidden, cap, cfg.tokens, topk_run, **_opts(args))
        else:
            nvm.gate_up_silu_ws(x, g, u, bufs.act, bufs.expert_offsets,
                                bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count,
                                cfg.inter, cfg.hidden, cap, cfg.tokens, topk_run, experts_run, ws,
                                **_opts(args))
    with torch.cuda.graph(gu_graph, stream=stream):
        for lay in layers:
            gate_up(lay)
    reps = max(3, min(2000, int(200.0 / max(0.7 * ms_per_step * len(layers), 1e-4))))
    with torch.cuda.stream(stream):
        gu_graph.replay()
        ev0.record(stream)
        for _ in range(reps):
            gu_graph.replay()
        ev1.record(stream)
    torch.cuda.synchronize(dev)
    gu_ms = ev0.elapsed_time(ev1) / (reps * len(layers))
    gu_bytes = 2 * (active + (1 if args.shared else 0)) * per_expert
    # Stored traffic describes the default launch of the captured workload only.
    default_launch = not _overrides(args) and not args.shared and not any(
        v for k, v in _opts(args).items())

    def traffic(kernel):
        t = ncu_traffic(cfg.name, kernel) if default_launch else None
        out = {"traffic": t, "traffic_source_hash": kernel_source_hash(kernel)}
        if t is not None and (cfg.name, kernel) in NCU_TRAFFIC_SCALED:
            out["traffic_scaled"] = NCU_TRAFFIC_SCALED[(cfg.name, kernel)]
        return out

    gu_flops = 2.0 * 2 * pairs_run * cfg.hidden * cfg.inter
    rows = _tc_rows(args, cfg.tokens, pairs_run, experts_run) if tc else 0
    if prefill:
        achieved = gu_flops / (gu_ms * 1e-3) / 1e12
        roofline = {"kernel": f"nvfp4_moe_gate_up_silu_ws ({_tc_kernel_name(rows)})", "bound": "tensor",
                    "achieved": achieved, "peak": tflops, "unit": "TFLOP/s",
                    "frac": achieved / tflops, "peak_source": f"{peak_kind} bf16 burst",
                    "algorithmic_flops_per_launch": gu_flops, "launch_ms": gu_ms,
                    **traffic("tcgen05")}
    else:
        achieved = gu_bytes / (gu_ms * 1e-3) / 1e9
        roofline = {"kernel": f"nvfp4_moe_gate_up_silu_ws ({_tc_kernel_name(rows)})" if tc else
                    "nvfp4_moe_gate_up_silu (register-fed mma.sync)", "bound": "hbm",
                    "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                    "peak_source": f"{peak_kind} HBM copy", "algorithmic_bytes_per_launch": gu_bytes,
                    "launch_ms": gu_ms, **traffic("tcgen05" if tc else "mma.sync")}

    e2e = None if args.no_e2e else run_e2e(layers, prob, bufs, ws, dev, stream, steps, warmup, args,
                                            world, overlap=ms_per_step >= E2E_OVERLAP_MIN_MS)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(prob, shared=args.shared)

    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16-mma/f32-acc", "data": "synthetic",
        "config": {"workload": cfg.name + ("+shared" if args.shared else "")
                   + (" (reduced: experts/tokens overridden)" if _overrides(args) else ""),
                   "hidden": cfg.hidden, "inter": cfg.inter,
                   "experts": cfg.experts, "topk": cfg.topk, "tokens": cfg.tokens,
                   "router": cfg.router, "active_experts": active,
                   "shared_expert": ({"rows_per_table_entry": base.rows_per_shared_slot(cfg.tokens),
                                      "table_entries": slots} if args.shared else None),
                   "path": (f"tcgen05-pair-nt{rows}" if rows in (32, 192, 256) else f"tcgen05-nt{rows}")
                           if tc else "mma.sync",
                   "weight_replicas": len(layers),
                   "l2": f"weights rotate over {len(layers)} device replicas; "
                         f"{len(layers)} x {routed_bytes/1e6:.1f} MB routed >= 4 x L2 ({l2/1e6:.0f} MB)"
                         if len(layers) > 1 else f"routed bytes {routed_bytes/1e6:.0f} MB > 4 x L2",
                   "parallelism": f"replicas x{world}"},
        "median_step": {"ms": median_ms, "tokens_per_s": world * cfg.tokens / (median_ms * 1e-3),
                        "replays": n_med,
                        "how": "median of per-replay CUDA-event times of single-step graphs"},
        "timed_region": f"one replay of a CUDA graph of exactly {steps} layer forwards "
                        f"(step i on weight replica i mod {len(layers)})",
        "routed_weight_gbs": {"value": routed_gbs, "peak": hbm, "frac": routed_gbs / hbm,
                              "bytes_per_step": routed_bytes},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        # [append_shared,] route_sort, [pack, tensor maps,] gate+up, [pack, tensor maps,]
        # down, blend
        "gpu_launches": ((8 if tc else 4) + (1 if args.shared else 0)) * steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        del g_steps, g_one, gu_graph
        dist.destroy_process_group()


def _op_traffic(op, workload):
    """ncu DRAM bytes of one launch of a load-time op's kernel, or None when absent
    or taken from other sources."""
    entry = NCU_OP_TRAFFIC_BYTES.get((op, workload))
    kernel = {"check_scales": "check_scales", "twins": "transpose_u8"}.get(op)
    if entry is None or kernel is None or entry[1] != kernel_source_hash(kernel):
        return None
    return entry[0]


def _overrides(args):
    """Reduced-case overrides (profiling): expert and token counts."""
    out = {}
    if args.experts:
        out["experts"] = args.experts
    if args.tokens:
        out["tokens"] = args.tokens
    return out


def _opts(args):
    return dict(path=args.path, split=args.split, tiles=args.tiles, depth=args.depth,
                staging=args.staging)


def _tc_path(args, cfg, pairs, experts):
    """Whether the projections take the tcgen05 path (the library's rule for
    the workspace calls: widths divisible by 128 / 256, and path 2, or path 0
    with at least 2 routed rows per expert on average)."""
    if args.path == 1 or cfg.inter % 128 or cfg.hidden % 256:
        return False
    return args.path == 2 or pairs >= 2 * experts


def _uses_prefill(args, pairs, experts):
    """Many rows per expert: a dense contraction, tensor-bound (else HBM-bound)."""
    return (pairs + experts - 1) // experts > 16


def _tc_rows(args, tokens, pairs, experts):
    """Token rows per pass of the tcgen05 kernels (the library's rule): 16 / 128 on
    the one-CTA kernel, 32 / 192 on the CTA-pair kernel."""
    if args.tiles:
        return args.tiles * 8
    mean = (pairs + experts - 1) // experts
    if mean > 16:
        return 256
    return 32 if tokens > 16 and mean <= 4 else 16


def _tc_kernel_name(rows):
    if rows == 256:
        return "tcgen05 CTA pair, 256-row passes, A in shared memory"
    return (f"tcgen05 CTA pair, {rows}-row passes" if rows in (32, 192)
            else f"tcgen05 one CTA, {rows}-row passes")


# Device step time from which the end-to-end loop overlaps its copies with the
# neighbouring steps' forwards; below it the host's per-step cost of the
# three-stream schedule exceeds the copy time it hides (measured: decode M=1
# 20.8 k -> 15.4 k tokens/s overlapped, prefill 1.21 M -> 2.33 M).
E2E_OVERLAP_MIN_MS = 0.15


def run_e2e(layers, prob, bufs, ws, dev, stream, steps, warmup, args, world, overlap):
    """Same metric through the public API from pinned host buffers: every step
    copies its inputs (x, topk_ids, topk_weights) host->device, runs the forward
    and copies its FP32 output device->host, all inside the timed region.  With
    `overlap`, as a serving loop would, the copies run on their own streams,
    overlapping the neighbouring steps' forwards (inputs and outputs
    double-buffered; events order each buffer's reuse); without, all three run
    in order on one stream."""
    import torch
    cfg = prob.cfg
    # The step's inputs staged in one pinned block (x | topk_ids | topk_weights,
    # each 256-byte aligned) and copied with one host->device copy.
    x_np = prob.x_bf16.view(np.int16)
    ids_np = np.ascontiguousarray(prob.topk_ids)
    w_np = np.ascontiguousarray(prob.topk_weights)
    al = lambda v: (v + 255) // 256 * 256
    sizes = [x_np.nbytes, ids_np.nbytes, w_np.nbytes]
    offs = [0, al(sizes[0]), al(sizes[0]) + al(sizes[1])]
    total = offs[2] + al(sizes[2])
    hblock = torch.empty(total, dtype=torch.uint8).pin_memory()
    hblock[offs[0]:offs[0] + sizes[0]].copy_(torch.from_numpy(x_np.view(np.uint8).reshape(-1)))
    hblock[offs[1]:offs[1] + sizes[1]].copy_(torch.from_numpy(ids_np.view(np.uint8).reshape(-1)))
    hblock[offs[2]:offs[2] + sizes[2]].copy_(torch.from_numpy(w_np.view(np.uint8).reshape(-1)))

    class Slot:
        def __init__(self, out_bufs):
            self.dblock = torch.empty(total, dtype=torch.uint8, device=dev)
            self.dx = self.dblock[offs[0]:offs[0] + sizes[0]].view(torch.bfloat16).view(cfg.tokens, cfg.hidden)
            self.dids = self.dblock[offs[1]:offs[1] + sizes[1]].view(torch.int32).view(cfg.tokens, cfg.topk)
            self.dw = self.dblock[offs[2]:offs[2] + sizes[2]].view(torch.float32).view(cfg.tokens, cfg.topk)
            self.bufs = out_bufs
            self.hout = torch.empty((cfg.tokens, cfg.hidden), dtype=torch.float32).pin_memory()
            self.ev_in = torch.cuda.Event()     # inputs on the device
            self.ev_fwd = torch.cuda.Event()    # forward done (inputs free, output ready)
            self.ev_out = torch.cuda.Event()    # output on the host (output buffers free)

    slots = [Slot(bufs), Slot(layers[0].buffers(cfg.tokens))]
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    n = max(1, min(steps, 2000))
    started = [False, False]

    def run_serial(count):
        sl = slots[0]
        with torch.cuda.stream(stream):  # one stream context for the loop: host-bound steps
            for i in range(count):
                sl.dblock.copy_(hblock, non_blocking=True)
                layers[i % len(layers)].forward(sl.dx, sl.dids, sl.dw, sl.bufs, workspace=ws,
                                                **_opts(args))
                sl.hout.copy_(sl.bufs.out[: cfg.tokens], non_blocking=True)

    def one_overlap(i):
        sl = slots[i % 2]
        if started[i % 2]:
            s_in.wait_event(sl.ev_fwd)          # the forward two steps back has read dblock
            stream.wait_event(sl.ev_out)        # ... and its output has left the device
        started[i % 2] = True
        with torch.cuda.stream(s_in):
            sl.dblock.copy_(hblock, non_blocking=True)
            sl.ev_in.record(s_in)
        stream.wait_event(sl.ev_in)
        with torch.cuda.stream(stream):
            layers[i % len(layers)].forward(sl.dx, sl.dids, sl.dw, sl.bufs, workspace=ws, **_opts(args))
            sl.ev_fwd.record(stream)
        s_out.wait_event(sl.ev_fwd)
        with torch.cuda.stream(s_out):
            sl.hout.copy_(sl.bufs.out[: cfg.tokens], non_blocking=True)
            sl.ev_out.record(s_out)

    def run_overlap(count):
        for i in range(count):
            one_overlap(i)
        for k, sl in enumerate(slots):  # both slots' outputs are on the host
            if started[k]:
                stream.wait_event(sl.ev_out)

    run = run_overlap if overlap else run_serial

    run(max(3, warmup))
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    s_in.wait_event(ev0)
    run(n)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms = reduce_max(ev0.elapsed_time(ev1))
    # The streamed result is the forward's: the last step's host copy against a
    # fresh forward of the same inputs (same kernels, deterministic: bit-equal).
    last = slots[(n - 1) % 2] if overlap else slots[0]
    with torch.cuda.stream(stream):
        layers[(n - 1) % len(layers)].forward(last.dx, last.dids, last.dw, bufs, workspace=ws, **_opts(args))
    stream.synchronize()
    if not torch.equal(last.hout, bufs.out[: cfg.tokens].cpu()):
        raise RuntimeError("end-to-end result differs from a plain forward of the same inputs")
    h2d = total
    d2h = last.hout.numel() * 4
    return {"value": world * cfg.tokens * n / (ms * 1e-3), "unit": "tokens/s", "steps": n,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "schedule": "overlapped" if overlap else "serial",
            "api": "NVFP4MoE.forward (one nvfp4_moe_forward call per step, eager launches); "
                   "inputs staged in one pinned block; per step one H2D and one D2H copy, "
                   + ("on copy streams overlapping the neighbouring steps' forwards "
                      "(double-buffered)" if overlap else "in order with the forward on one stream")}


# --------------------------------------------------------------------------- #
# The CPU oracle as baseline / reference arm
# --------------------------------------------------------------------------- #

def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def _oracle_sample(prob):
    """A bounded slice of the workload for the oracle: at most 2 tokens' full forward."""
    from workloads import make_problem
    import dataclasses
    cfg = prob.cfg
    m = min(cfg.tokens, 2 if cfg.tokens > 1 else 1)
    sub = make_problem(cfg)
    sub.x_bf16 = prob.x_bf16[:m].copy()
    sub.topk_ids = prob.topk_ids[:m].copy()
    sub.topk_weights = prob.topk_weights[:m].copy()
    sub.cfg = dataclasses.replace(cfg, tokens=m)
    return sub


def _oracle_step(sub, shared=None):
    import oracle as orc
    cfg = sub.cfg
    fns = [lambda e, mm=mm: sub.expert_weight(mm, e, cache=True) for mm in (0, 1, 2)]
    if shared is None:
        orc.moe_forward(sub.x_bf16, sub.topk_ids, sub.topk_weights, cfg.experts, *fns,
                        hidden=cfg.hidden, inter=cfg.inter)
    else:
        orc.moe_forward_shared(sub.x_bf16, sub.topk_ids, sub.topk_weights, cfg.experts, *fns,
                               hidden=cfg.hidden, inter=cfg.inter, shared=shared)


def _shared_weights(sub, shared: bool):
    return tuple(sub.shared_weight(mm) for mm in (0, 1, 2)) if shared else None


def cpu_baseline(prob, budget_s=12.0, shared=False):
    sub = _oracle_sample(prob)
    sh = _shared_weights(sub, shared)
    _oracle_step(sub, sh)  # draws (and caches) the sample's expert bytes
    t0 = time.perf_counter()
    n = 0
    while True:
        _oracle_step(sub, sh)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": sub.cfg.tokens * n / dt, "unit": "tokens/s", "cores": _oracle_threads(),
            "kind": "oracle",
            "sample": f"{n} fp64 oracle forwards of the first {sub.cfg.tokens} token(s) of "
                      f"{prob.cfg.name}{' with the shared expert' if shared else ''} (route sort, "
                      f"dequantise the experts, gate+up SiLU, down, blend), weight bytes "
                      f"pre-drawn, {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from workloads import make_problem
    prob = make_problem(args.config)
    steps = args.steps if args.steps is not None else 5
    warmup = max(args.warmup, 3)
    sub = _oracle_sample(prob)
    sh = _shared_weights(sub, args.shared)
    for _ in range(min(warmup, 1) if steps > 20 else warmup):
        _oracle_step(sub, sh)
    t0 = time.perf_counter()
    for _ in range(steps):
        _oracle_step(sub, sh)
    dt = time.perf_counter() - t0
    value = sub.cfg.tokens * steps / dt
    cores = _oracle_threads()
    sample = (f"each step: fp64 oracle forward of the first {sub.cfg.tokens} token(s) of "
              f"{prob.cfg.name}{' with the shared expert' if args.shared else ''}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": 0, "steps": steps, "warmup": warmup, "ms_per_step": dt * 1e3 / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": prob.cfg.name + ("+shared" if args.shared else ""), "hidden": prob.cfg.hidden, "inter": prob.cfg.inter,
                       "experts": prob.cfg.experts, "topk": prob.cfg.topk, "tokens": prob.cfg.tokens},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_load_op(args, rank, world, local):
    """A load-time op over the gate, up and down weights of every expert of the
    workload, one library call per projection: nvfp4_moe_check_scales (an
    HBM-bound byte scan of the scale tables) or nvfp4_moe_shard_nvfp4 (rank 0's
    tensor-parallel shard: gate / up by rows, down by K; bytes read + written)."""
    import torch
    import nvfp4_weight_quantized_moe_b200 as nvm
    from workloads import make_problem
    from workloads.device import upload_layer

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    prob = make_problem(args.config, **_overrides(args))
    cfg = prob.cfg
    layer = upload_layer(prob, dev)
    projs = (layer.gate, layer.up, layer.down)
    bad = torch.zeros(3, cfg.experts, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    shard = args.op == "shard"
    twins = args.op == "twins"
    if twins:
        tw_out = [(torch.empty((cfg.hidden // 2, 2 * cfg.inter), dtype=torch.uint8, device=dev),
                   torch.empty((cfg.hidden // 16, 2 * cfg.inter), dtype=torch.uint8, device=dev))
                  for _ in range(cfg.experts)]
        moved = 2 * 2 * cfg.experts * (layer.gate.packed[0].numel() + layer.gate.scale[0].numel())
    elif shard:
        kinds = (nvm.SHARD_COLUMN, nvm.SHARD_COLUMN, nvm.SHARD_ROW)
        outs = [nvm.shard_nvfp4(p.packed, p.scale, kd, 0, args.tp) for p, kd in zip(projs, kinds)]
        moved = 2 * sum(o[0].numel() + o[1].numel() for o in outs)  # read + written
    else:
        moved = sum(p.scale.numel() for p in projs)
    scale_bytes = moved

    def one():
        if twins:
            for e in range(cfg.experts):
                nvm.transpose_concat_into(
                    [(layer.gate.packed[e], layer.gate.scale[e]), (layer.up.packed[e], layer.up.scale[e])],
                    16, tw_out[e][0], tw_out[e][1], stream=stream)
            return
        for i, p in enumerate(projs):
            if shard:
                nvm.shard_nvfp4_into(p.packed, p.scale, kinds[i], 0, args.tp, outs[i][0],
                                     outs[i][1], stream=stream)
            else:
                nvm.check_scales(p.tables, cfg.experts, p.n, p.k, bad[i], stream=stream)

    steps = args.steps if args.steps is not None else 200
    warmup = max(args.warmup, 3)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one()
    stream.synchronize()
    if int(bad.sum().item()) != 0:
        raise RuntimeError("generated scales reported invalid")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one()
    sampler = ClockSampler(local)
    sampler.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    sampler.mark(True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(steps):
            g.replay()
        ev1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark(False)
    clocks = sampler.stop()
    ms = ev0.elapsed_time(ev1) / steps
    hbm, _, _, peak_kind = measured_peaks()
    gbs = scale_bytes / (ms * 1e-3) / 1e9
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    what = (f"NVFP4 tensor-parallel shard GB/s (load time, tp={args.tp}, read + written)" if shard
            else "NVFP4 gate|up transposed twins GB/s (load time, read + written)" if twins
            else "NVFP4 block-scale check GB/s (load time)")
    line = {
        "metric": what, "value": gbs, "unit": "GB/s",
        "n_gpus": 1, "steps": steps, "warmup": warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": cfg.name + (" weights" if shard or twins else " scale tables"),
                   "experts": cfg.experts, "bytes_per_step": scale_bytes,
                   "l2": f"three projections, {scale_bytes / 3e6:.0f} MB moved each, "
                         f"L2 {l2 / 1e6:.0f} MB"},
        "roofline": {"kernel": "shard_copy_kernel" if shard else "transpose_u8_kernel" if twins
                     else "check_scales_kernel",
                     "bound": "hbm", "achieved": gbs, "peak": hbm,
                     "unit": "GB/s", "frac": gbs / hbm, "peak_source": f"{peak_kind} HBM copy",
                     "traffic": _op_traffic(args.op, cfg.name),
                     "traffic_unit": "bytes per launch (one projection's scale table; one "
                                     "transposed packed part)"},
        "gpu_launches": (4 * cfg.experts if twins else 6 if shard else 3) * steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_info()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.op in ("check_scales", "shard", "twins"):
        run_load_op(args, rank, world, local)
        return
    run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
