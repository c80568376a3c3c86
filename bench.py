"""Benchmark of the routed-MoE expert pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--only NAME] [--impl ours|reference]
                    [--seed S] [--nvtx]

A step is one pass of the whole hot path — router logits + top-k + gates,
slot lookup + miss list, expert FFNs, combine — over one batch of synthetic
tokens at the workload's shapes.  Rank 0 prints one JSON line.

The headline (`value`, `e2e`, `roofline`, `cpu_baseline`) is the one-layer
decode workload: 4 tokens (1 + 3 MTP drafts), 512 experts, top-10 + shared,
Q2_32, 320 of 512 experts resident.  The same line carries one keyed object
per other workload, each measured the same way:
  prefill    one layer, 2,048 tokens, Q2_32, all resident, Zipf(0.8) loads
  decode48   48 chained layers, 1 token, Q3_32, 7,948 resident slots
  prefill48  48 chained layers, 4,096 tokens, Q3_S256, all 24,576 experts resident
  decode_coder, prefill_coder
             the decode and prefill workloads at the 256-expert Coder shape, all resident

Timing: CUDA graphs of whole steps are replayed until exactly K steps ran;
barrier + synchronize on both sides; CUDA events on the launching stream; max
over ranks.  L2 (126 MB) is defeated by rotating over replicas of the expert
pool, router weights and token batches for the one-layer workloads; the
48-layer workloads read 19 GB / 50 GB of experts per step.  Per-kernel
durations come from external event nodes inside the same graph; each roofline
object also gives their p10 / p50 / p90.  --seed replaces every workload's
seed (weights, router, tokens) to report other draws of the same recipe;
--nvtx puts NVTX ranges around each workload and each timed region.
"""
from __future__ import annotations

import argparse
import contextlib
import dataclasses
import gc
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_expert_ffn_route_b200 import configs, moe, synth  # noqa: E402

METRIC = "MoE expert-pass tokens/s per layer"
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
EXTRA = ["prefill", "decode48", "prefill48", "decode_coder", "prefill_coder"]
# kernels per layer and step: the one-call decode layer (T <= 8) 1; decode as
# three calls: route 1, expert pass 1, combine 1; prefill route 3 (norms, tensor-core logits, selection), expert pass 6 (3
# plan, gather, 2 GEMMs), combine 1
LAUNCHES = {"layer": 1, "decode": 3, "prefill": 10}


def _cfg(name, args):
    """The workload's config, with --seed (when given) for every synthetic input."""
    cfg = configs.CONFIGS[name]
    return cfg if getattr(args, "seed", None) is None else dataclasses.replace(cfg, seed=args.seed)


def _pct_us(ms):
    """p10 / p50 / p90 of per-launch durations (ms) in microseconds."""
    return [round(float(np.percentile(ms, q)) * 1e3, 3) for q in (10, 50, 90)]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _traffic(kind):
    """DRAM bytes per launch from the committed ncu capture of this workload's
    dominant launch (keyed by workload name), or None when there is none or the
    kernel's sources changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            e = json.load(f)[kind]
        h = hashlib.sha256()
        for src in e["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != e["sha256"]:
            return None, None
        return int(e["bytes_per_launch"]), e["covers"]
    except (OSError, KeyError, ValueError):
        return None, None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        # raw samples: a scratch file (the summary goes into the JSON line);
        # MOE_BENCH_CLOCKS_DIR keeps them somewhere else
        out_dir = os.environ.get("MOE_BENCH_CLOCKS_DIR", tempfile.gettempdir())
        self.path = os.path.join(out_dir, f"moe_bench_clocks_rank{index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1])); mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names[1:], parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, ws: int, device) -> float:
    """The largest of every rank's value (each rank calls it at the same point;
    with one rank, the value itself)."""
    if ws <= 1:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _graph_of(fn, n_steps, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n_steps):
            fn(i)
    return g


def _divisor_at_most(K, cap):
    for g in range(min(K, cap), 0, -1):
        if K % g == 0:
            return g
    return 1


def _barrier(ws_):
    torch.cuda.synchronize()
    if ws_ > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


NVTX = False            # --nvtx: host ranges around each workload and each timed region


@contextlib.contextmanager
def _nvtx(name):
    """An NVTX range (for `ncu --nvtx --nvtx-include`) when --nvtx is given."""
    if NVTX:
        torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        if NVTX:
            torch.cuda.nvtx.range_pop()


def _timed_replays(graph, n, stream, ws_, dev, local, clocks=True):
    """Replay `graph` n times on `stream` between barriers; returns (max-over-ranks
    ms, clock summary)."""
    _barrier(ws_)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) if clocks else _NoClock() as clk, torch.cuda.stream(stream), _nvtx("timed"):
        t0.record(stream)
        for _ in range(n):
            graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    _barrier(ws_)
    return max_over_ranks(t0.elapsed_time(t1), ws_, dev), clk.summary()


class _NoClock:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass

    def summary(self):
        return None


def _roofline(kind, per_launch, avg_ms, peaks, traffic_kind):
    hbm, tf, tf_sus, peak_kind = peaks
    traffic, covers = _traffic(traffic_kind)
    if kind == "hbm":
        achieved = per_launch / (avg_ms / 1e3) / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": traffic, "traffic_covers": covers,
                "peak_kind": f"{peak_kind} copy bandwidth", "algorithmic_bytes_per_launch": round(per_launch),
                "avg_launch_us": round(avg_ms * 1e3, 3)}
    achieved = per_launch / (avg_ms / 1e3) / 1e12
    # the expert pass is timed as a ~1 ms kernel sequence inside sub-second
    # regions: the burst GEMM figure is its denominator (sustained for context)
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": tf, "unit": "TFLOP/s",
            "frac": round(achieved / tf, 4), "frac_of_sustained": round(achieved / tf_sus, 4), "traffic": traffic,
            "traffic_covers": covers, "peak_kind": f"{peak_kind} bf16 burst (sustained {tf_sus})",
            "algorithmic_flops_per_launch": round(per_launch), "avg_launch_us": round(avg_ms * 1e3, 3)}


def _fp8_variant(layers, xs, R, G, K, k, T, D, stream, ev, ws_, dev, local, fwd_flops, peaks, traffic_key):
    """The same prefill steps with the e4m3-operand expert pass
    (moe_expert_forward_fp8): step time and the expert pass against the e4m3
    tensor peak (the measured bf16 peak x 2, the nominal dense ratio)."""
    with torch.cuda.stream(stream):
        for r in range(R):
            layers[r](xs[r], stream=stream, fp8=True)          # allocates each layer's e4m3 workspace
    torch.cuda.synchronize()

    def fp8_step(i, events=False):
        lay = layers[i % R]
        moe.moe_route_topk(xs[i % R], lay.Wr, lay.bias, k, lay.ids, lay.gates, lay.route_ws, stream=stream)
        if events:
            ev[i][0].record(stream)
        moe.moe_expert_forward_fp8(lay.pool, lay.slot_table, xs[i % R], lay.ids, k, lay.expert_out, lay.miss_list,
                                   lay.miss_count, lay.ws_fp8, stream=stream)
        if events:
            ev[i][1].record(stream)
        moe.moe_combine(lay.expert_out, lay.gates, T, D, k, lay.out, stream=stream)

    g8 = _graph_of(fp8_step, G, stream)
    g8e = _graph_of(lambda i: fp8_step(i, True), G, stream)
    with torch.cuda.stream(stream):
        g8.replay()
        g8e.replay()
    ms8, _ = _timed_replays(g8, K // G, stream, ws_, dev, local, clocks=False)
    _timed_replays(g8e, K // G, stream, ws_, dev, local, clocks=False)
    fwd8 = float(np.mean([ev[i][0].elapsed_time(ev[i][1]) for i in range(G)]))
    hbm, tf, tf_sus, kind = peaks
    roof8 = _roofline("tensor", float(np.mean([fwd_flops[i % R] for i in range(G)])), fwd8,
                      (hbm, round(2 * tf, 1), round(2 * tf_sus, 1), kind), traffic_key)
    roof8["peak_kind"] = f"measured bf16 burst x 2 (e4m3 nominal dense ratio); sustained {round(2 * tf_sus, 1)}"
    roof8["kernel"] = "moe_expert_forward_fp8 (plan + e4m3 gather + tcgen05 kind::f8f6f4 grouped GEMMs)"
    del g8, g8e
    return {"value": round(ws_ * T * K / (ms8 / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms8 / K, 6),
            "dtype": "e4m3 operands (weights x64, x, h), fp32 accumulate; lossy, see tests/test_gpu_fp8.py",
            "roofline": roof8}


# ---------------------------------------------------------------- one-layer workloads
def bench_layer(name, K, W, ws_, dev, local, args, with_cpu):
    cfg = _cfg(name, args)
    T, D, F, E, k = cfg.T, cfg.D, cfg.F, cfg.E, cfg.k
    wl = configs.build(cfg, device=dev)
    L0 = wl.layers[0]
    slot_bytes = wl.pool.slot_bytes
    pool_bytes = wl.pool.n_slots * slot_bytes
    # decode touches ~(U+1) experts + Wr (~65 MB) per step: 8 replicas put ~450 MB
    # of other traffic between two uses of one replica (L2 is 126 MB)
    R = args.replicas or (8 if T <= 8 else 2)
    pools, Wrs, xs = [], [], []
    for r in range(R):
        if r == 0:
            pools.append(wl.pool)
            Wrs.append(L0.Wr)
        else:
            pools.append(synth.PoolData(wl.pool.fmt, D, F, wl.pool.n_slots, wl.pool.codes.clone(),
                                        wl.pool.scales.clone(), wl.pool.stride_codes, wl.pool.stride_scales))
            Wrs.append(L0.Wr.clone())
        xs.append(synth.hidden(T, D, cfg.seed, stream=100 + r, device=dev))
    layers = [moe.Layer(pools[r], L0.shared_slot, L0.slot_table, Wrs[r], L0.bias, k, T, device=dev)
              for r in range(R)]
    stream = torch.cuda.Stream(device=dev)
    table = L0.slot_table.cpu().numpy()
    with torch.cuda.stream(stream):
        for r in range(R):
            layers[r](xs[r], stream=stream)
    torch.cuda.synchronize()
    u_hit, hits = [], []
    for r in range(R):
        sl = table[layers[r].ids.cpu().numpy()]
        u_hit.append(len(np.unique(sl[sl >= 0])))
        hits.append(float((sl >= 0).mean()))
    x_bytes = T * D * 2
    wr_bytes = E * D * 2
    fwd_bytes = [(u + 1) * slot_bytes + x_bytes for u in u_hit]         # expert weights read + x
    step_bytes = [fb + wr_bytes + x_bytes for fb in fwd_bytes]           # + router weights + out
    # the decode step is the one-call layer (routing, expert pass and combine
    # in one kernel): its algorithmic bytes are the whole step's
    fused = T <= 8 and layers[0].layer_ws is not None
    # algorithmic FLOPs of the expert FFNs: every resident (token, rank) row and
    # every token's shared-expert row costs gate + up + down = 3 * 2 * D * F
    fwd_flops = [(h * T * k + T) * 6.0 * D * F for h in hits]

    G = _divisor_at_most(K, 512 if T <= 8 else 64)
    ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(G)]

    def step(i, events=False):
        lay = layers[i % R]
        if fused:
            if events:
                ev[i][0].record(stream)
            lay.fused(xs[i % R], stream=stream)
            if events:
                ev[i][1].record(stream)
            return
        three_calls(i, events)

    def three_calls(i, events=False):
        lay = layers[i % R]
        moe.moe_route_topk(xs[i % R], lay.Wr, lay.bias, k, lay.ids, lay.gates, lay.route_ws, stream=stream)
        if events:
            ev[i][0].record(stream)
        moe.moe_expert_forward(lay.pool, lay.slot_table, xs[i % R], lay.ids, k, lay.expert_out, lay.miss_list,
                               lay.miss_count, lay.ws, stream=stream)
        if events:
            ev[i][1].record(stream)
        moe.moe_combine(lay.expert_out, lay.gates, T, D, k, lay.out, stream=stream)

    # the throughput graph has no event nodes: an event recorded between two
    # kernels ends the programmatic-launch overlap of the second with the first
    graph = _graph_of(step, G, stream)
    graph_ev = _graph_of(lambda i: step(i, True), G, stream)
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-W // G))):
            graph.replay()
            graph_ev.replay()
    ms, clocks = _timed_replays(graph, K // G, stream, ws_, dev, local)
    # the dominant kernel's own duration: the same steps with an event pair
    # around each moe_layer_forward (decode) or moe_expert_forward (prefill)
    # launch, so launched without the overlap
    _timed_replays(graph_ev, K // G, stream, ws_, dev, local, clocks=False)
    fwd_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(G)]
    value = ws_ * T * K / (ms / 1e3)
    fwd_avg_ms = float(np.mean(fwd_ms))
    peaks = _peaks()
    three = None
    if fused:
        # the same layer as three calls (router, expert pass, combine), for comparison
        g3 = _graph_of(three_calls, G, stream)
        with torch.cuda.stream(stream):
            g3.replay()
        ms3, _ = _timed_replays(g3, K // G, stream, ws_, dev, local, clocks=False)
        three = {"ms_per_step": round(ms3 / K, 6), "value": round(ws_ * T * K / (ms3 / 1e3), 1),
                 "calls": "moe_route_topk + moe_expert_forward + moe_combine"}
        del g3
        roof = _roofline("hbm", float(np.mean([step_bytes[i % R] for i in range(G)])), fwd_avg_ms, peaks, name)
        roof["kernel"] = ("moe_layer_forward (decode_ffn_kernel, one-call layer: logits + top-k, gate|up and down "
                          "dequant-GEMV, combine); bytes = Wr + resident experts read + x + out")
    elif T <= 8:
        roof = _roofline("hbm", float(np.mean([fwd_bytes[i % R] for i in range(G)])), fwd_avg_ms, peaks,
                         name + "_three_calls")
        roof["kernel"] = "moe_expert_forward (decode_ffn_kernel: gate|up + down dequant-GEMV)"
    else:
        roof = _roofline("tensor", float(np.mean([fwd_flops[i % R] for i in range(G)])), fwd_avg_ms, peaks, name)
        roof["kernel"] = "moe_expert_forward (plan + gather + tcgen05 gate|up and down grouped GEMMs)"
    roof["launch_us_p10_p50_p90"] = _pct_us(fwd_ms)

    # end to end through the public API: pinned host input -> device, the layer
    # call(s), device -> pinned host output, every step.  The copies run on a
    # copy stream, pipelined with the neighbouring steps' compute: step i's
    # input is copied in during step i - 1 and its output copied out during
    # step i + 1 (buffers rotate over R replicas; step i's layer waits for the
    # copy-out of step i - R, the last reader of its output buffer)
    xh = [torch.empty(T, D, dtype=torch.bfloat16).pin_memory() for _ in range(R)]
    oh = [torch.empty(T, D, dtype=torch.bfloat16).pin_memory() for _ in range(R)]
    for r in range(R):
        xh[r].copy_(xs[r].cpu())
    xd = [torch.empty(T, D, dtype=torch.bfloat16, device=dev) for _ in range(R)]
    copy_stream = torch.cuda.Stream(device=dev)
    Ge = _divisor_at_most(K, 256 if T <= 8 else 32)
    ev_in = [torch.cuda.Event() for _ in range(Ge)]
    ev_done = [torch.cuda.Event() for _ in range(Ge)]
    ev_out = [torch.cuda.Event() for _ in range(Ge)]

    def e2e_steps():
        copy_stream.wait_stream(stream)
        with torch.cuda.stream(copy_stream):
            xd[0].copy_(xh[0], non_blocking=True)
            ev_in[0].record(copy_stream)
        for i in range(Ge):
            r = i % R
            if i + 1 < Ge:
                with torch.cuda.stream(copy_stream):
                    xd[(i + 1) % R].copy_(xh[(i + 1) % R], non_blocking=True)
                    ev_in[i + 1].record(copy_stream)
            stream.wait_event(ev_in[i])
            if i >= R:
                stream.wait_event(ev_out[i - R])
            if fused:
                layers[r].fused(xd[r], stream=stream)
            else:
                layers[r](xd[r], stream=stream)
            ev_done[i].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev_done[i])
                oh[r].copy_(layers[r].out, non_blocking=True)
                ev_out[i].record(copy_stream)
        stream.wait_stream(copy_stream)

    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        e2e_steps()
    with torch.cuda.stream(stream):
        g2.replay()
    ems, _ = _timed_replays(g2, K // Ge, stream, ws_, dev, local, clocks=False)
    res = {
        "value": round(value, 1), "unit": "tokens/s", "ms_per_step": round(ms / K, 6), "steps": K,
        "workload": f"{cfg.name}: 1 layer, T={T}, D={D}, F={F}, E={E}, top-{k}+1 shared, "
                    f"{synth.FMT_NAMES[cfg.fmt]}, {int((table >= 0).sum())}/{E} resident",
        "l2": f"rotating {R} replicas of pool+Wr+x ({R * pool_bytes / 1e9:.2f} GB)",
        "e2e": {"value": round(ws_ * T * K / (ems / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": T * D * 2,
                "d2h_bytes_per_step": T * D * 2, "copies": "pinned host buffers, on a copy stream overlapping the "
                                                           "neighbouring steps' compute"},
        "gpu_launches": LAUNCHES["layer" if fused else ("decode" if T <= 8 else "prefill")] * K,
        "roofline": roof,
        "hit_rate": round(float(np.mean(hits)), 4), "u_hit_mean": round(float(np.mean(u_hit)), 2),
        "step_alg_bytes": round(float(np.mean(step_bytes))),
        "clocks": clocks,
    }
    if three is not None:
        res["three_calls"] = three
    if T > 8:
        res["fp8_variant"] = _fp8_variant(layers, xs, R, G, K, k, T, D, stream, ev, ws_, dev, local, fwd_flops, peaks,
                                          name + "_fp8")
    if T > 8:
        loads = np.bincount(layers[0].ids.cpu().numpy().ravel(), minlength=E)
        res["expert_loads"] = {"max": int(loads.max()), "zero": int((loads == 0).sum()),
                               "below_16": int((loads < 16).sum())}
    if with_cpu:
        res["cpu_baseline"] = cpu_baseline(cfg, wl, seconds=args.cpu_seconds)
    del layers, pools, Wrs, xs, graph, graph_ev, g2, wl
    return res


# ---------------------------------------------------------------- small verify batches
def bench_small_batches(ws_, dev, local, args, Ts=(1, 4, 5, 8, 9, 12, 16, 24, 25, 32, 64), K=64):
    """The decode layer's shapes at other batch sizes (MTP draft verification):
    per-step time and tokens/s of the three calls, and which expert-pass path
    ran (decode: T <= 24, tensor-core GEMV in launches of up to 8 tokens;
    prefill: T > 24, grouped GEMMs)."""
    cfg = _cfg("decode", args)
    wl = configs.build(cfg, device=dev, T=max(Ts))
    L0 = wl.layers[0]
    R = 8
    pools = [wl.pool] + [synth.PoolData(wl.pool.fmt, cfg.D, cfg.F, wl.pool.n_slots, wl.pool.codes.clone(),
                                        wl.pool.scales.clone(), wl.pool.stride_codes, wl.pool.stride_scales)
                         for _ in range(R - 1)]
    stream = torch.cuda.Stream(device=dev)
    out = {}
    for T in Ts:
        layers = [moe.Layer(pools[r], L0.shared_slot, L0.slot_table, L0.Wr, L0.bias, cfg.k, T, device=dev)
                  for r in range(R)]
        xs = [synth.hidden(T, cfg.D, cfg.seed, stream=600 + r, device=dev) for r in range(R)]

        def step(i):
            layers[i % R](xs[i % R], stream=stream)

        G = _divisor_at_most(K, 64)
        graph = _graph_of(step, G, stream)
        with torch.cuda.stream(stream):
            graph.replay()
        ms, _ = _timed_replays(graph, K // G, stream, ws_, dev, local, clocks=False)
        out[str(T)] = {"ms_per_step": round(ms / K, 5), "tokens_per_s": round(ws_ * T * K / (ms / 1e3), 1),
                       "expert_pass": (f"decode, {(T + 7) // 8} launches" if T > 8 else "decode") if T <= 24 else "prefill",
                       "router": "canonical CUDA-core" if T <= 24 else "tensor-core + canonical recheck"}
        if layers[0].layer_ws is not None:
            g1 = _graph_of(lambda i: layers[i % R].fused(xs[i % R], stream=stream), G, stream)
            with torch.cuda.stream(stream):
                g1.replay()
            ms1, _ = _timed_replays(g1, K // G, stream, ws_, dev, local, clocks=False)
            out[str(T)]["one_call"] = {"ms_per_step": round(ms1 / K, 5),
                                       "tokens_per_s": round(ws_ * T * K / (ms1 / 1e3), 1)}
            del g1
        del layers, xs, graph
    del pools, wl
    return {"workload": "decode layer shapes (D=3072, F=512, E=512, top-10+1, Q2_32, 320/512 resident), "
                        "T tokens per step, 8 rotating pool replicas", "by_T": out}


# ---------------------------------------------------------------- 48-layer chains
class ChainBuffers:
    """One set of buffers shared by every layer of a chain (the calls of a step
    run in stream order), plus one activation buffer per layer boundary."""

    def __init__(self, wl, dev):
        cfg = wl.cfg
        T, D, E, k = cfg.T, cfg.D, cfg.E, cfg.k
        self.pools = [moe.make_pool(wl.pool, L.shared_slot) for L in wl.layers]
        self.ids = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.gates = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.route_ws = moe.alloc_ws(moe.route_workspace_size(T, D, E, k), dev)
        self.ws = moe.alloc_ws(moe.workspace_size(T, D, cfg.F, E, k, cfg.fmt), dev)
        self.expert_out = moe.alloc_ws(moe.expert_out_size(T, D, k), dev)
        self.miss_list = torch.empty(T * k, 3, dtype=torch.int32, device=dev)
        self.miss_count = torch.zeros(1, dtype=torch.int32, device=dev)
        self.x = [torch.empty(T, D, dtype=torch.bfloat16, device=dev) for _ in range(len(wl.layers) + 1)]
        self.x[0].copy_(wl.x)
        n = moe.layer_workspace_size(T, D, cfg.F, E, k, cfg.fmt)     # the one-call layer (T <= 8)
        self.layer_ws = moe.alloc_ws(n, dev) if n else None

    def layer(self, wl, l, stream, ev=None, ids_out=None):
        cfg, L = wl.cfg, wl.layers[l]
        T, D, k = cfg.T, cfg.D, cfg.k
        if self.layer_ws is not None:
            if ev is not None:
                ev[0].record(stream)
            moe.moe_layer_forward(self.pools[l], L.slot_table, self.x[l], L.Wr, L.bias, k, self.ids, self.gates,
                                  self.expert_out, self.miss_list, self.miss_count, self.x[l + 1], self.layer_ws,
                                  residual=self.x[l], stream=stream)
            if ev is not None:
                ev[1].record(stream)
            if ids_out is not None:
                ids_out[l].copy_(self.ids)
            return
        moe.moe_route_topk(self.x[l], L.Wr, L.bias, k, self.ids, self.gates, self.route_ws, stream=stream)
        if ids_out is not None:
            ids_out[l].copy_(self.ids)
        if ev is not None:
            ev[0].record(stream)
        moe.moe_expert_forward(self.pools[l], L.slot_table, self.x[l], self.ids, k, self.expert_out,
                               self.miss_list, self.miss_count, self.ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        moe.moe_combine(self.expert_out, self.gates, T, D, k, self.x[l + 1], residual=self.x[l], stream=stream)


def bench_chain(name, K, W, ws_, dev, local, args, with_cpu):
    cfg = _cfg(name, args)
    T, D, F, E, k, NL = cfg.T, cfg.D, cfg.F, cfg.E, cfg.k, cfg.layers
    wl = configs.build(cfg, device=dev)
    buf = ChainBuffers(wl, dev)
    stream = torch.cuda.Stream(device=dev)
    # ids of every layer (the chain restarts from the same x each step, so they
    # are the same at every step): one untimed pass records them
    ids_all = [torch.empty(T, k, dtype=torch.int32, device=dev) for _ in range(NL)]
    with torch.cuda.stream(stream):
        for l in range(NL):
            buf.layer(wl, l, stream, ids_out=ids_all)
    torch.cuda.synchronize()
    slot_bytes = wl.pool.slot_bytes
    fwd_bytes, fwd_flops, hits, n_sel = [], [], 0, 0
    for l in range(NL):
        sl = wl.layers[l].slot_table.cpu().numpy()[ids_all[l].cpu().numpy()]
        u = len(np.unique(sl[sl >= 0]))
        fwd_bytes.append((u + 1) * slot_bytes + T * D * 2 + (E * D * 2 + T * D * 2 if buf.layer_ws is not None else 0))
        h = int((sl >= 0).sum())
        fwd_flops.append((h + T) * 6.0 * D * F)
        hits += h
        n_sel += sl.size
    ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(NL)]

    def step(i, events=False):
        for l in range(NL):
            buf.layer(wl, l, stream, ev=ev[l] if events else None)

    # no event nodes in the throughput graph (they end the programmatic-launch
    # overlap between kernels); a second graph times each expert pass
    graph = _graph_of(step, 1, stream)
    graph_ev = _graph_of(lambda i: step(i, True), 1, stream)
    with torch.cuda.stream(stream):
        for _ in range(W):
            graph.replay()
        graph_ev.replay()
    ms, clocks = _timed_replays(graph, K, stream, ws_, dev, local)
    _timed_replays(graph_ev, 1, stream, ws_, dev, local, clocks=False)
    fwd_ms = [ev[l][0].elapsed_time(ev[l][1]) for l in range(NL)]
    peaks = _peaks()
    if T <= 8:
        roof = _roofline("hbm", float(np.sum(fwd_bytes)) / NL, float(np.sum(fwd_ms)) / NL, peaks, name)
        roof["kernel"] = ("moe_layer_forward (decode_ffn_kernel, one-call layer), averaged over the 48 layers; "
                          "bytes = Wr + resident experts read + x + out")
    else:
        roof = _roofline("tensor", float(np.sum(fwd_flops)) / NL, float(np.sum(fwd_ms)) / NL, peaks, name)
        roof["kernel"] = "moe_expert_forward (plan + gather + tcgen05 GEMMs), averaged over the 48 layers"
    roof["launch_us_p10_p50_p90"] = _pct_us(fwd_ms)         # over the chain's layers
    # end to end: the first layer's input from pinned host memory, the last
    # layer's output back, every step
    xh = torch.empty(T, D, dtype=torch.bfloat16).pin_memory()
    oh = torch.empty(T, D, dtype=torch.bfloat16).pin_memory()
    xh.copy_(wl.x.cpu())

    def e2e_step(i):
        buf.x[0].copy_(xh, non_blocking=True)
        for l in range(NL):
            buf.layer(wl, l, stream)
        oh.copy_(buf.x[NL], non_blocking=True)

    g2 = _graph_of(e2e_step, 1, stream)
    with torch.cuda.stream(stream):
        g2.replay()
    ems, _ = _timed_replays(g2, K, stream, ws_, dev, local, clocks=False)
    res = {
        "value": round(ws_ * T * NL * K / (ms / 1e3), 1), "unit": "tokens/s (per layer)",
        "chain_tokens_per_s": round(ws_ * T * K / (ms / 1e3), 2), "ms_per_step": round(ms / K, 4), "steps": K,
        "workload": f"{cfg.name}: {NL} chained layers (x_l+1 = x_l + out_l), T={T}, D={D}, F={F}, E={E}, "
                    f"top-{k}+1 shared, {synth.FMT_NAMES[cfg.fmt]}, {wl.n_resident} resident slots",
        "l2": f"{NL} layers read {wl.pool.n_slots * slot_bytes / 1e9:.1f} GB of pool per step (> L2)",
        "e2e": {"value": round(ws_ * T * NL * K / (ems / 1e3), 1), "unit": "tokens/s (per layer)",
                "chain_tokens_per_s": round(ws_ * T * K / (ems / 1e3), 2), "h2d_bytes_per_step": T * D * 2,
                "d2h_bytes_per_step": T * D * 2},
        "gpu_launches": LAUNCHES["layer" if buf.layer_ws is not None else "prefill"] * NL * K,
        "roofline": roof,
        "hit_rate": round(hits / n_sel, 4),
        "clocks": clocks,
    }
    if with_cpu:
        res["cpu_baseline"] = cpu_baseline_chain(cfg, wl)
    del buf, graph, graph_ev, g2, wl
    return res


# ---------------------------------------------------------------- CPU baselines (the oracle)
def cpu_baseline(cfg, wl, seconds=10.0):
    """The oracle as it stands, on this host's cores, on whole steps of the same
    workload (all cores), plus one step on one thread."""
    from tests.harness import oracle_layer, u16
    ncores = os.cpu_count() or 1
    L0 = wl.layers[0]
    T = cfg.T
    sample_T = T if T <= 64 else 64
    n = 0
    t0 = time.time()
    while True:
        x = synth.hidden(sample_T, cfg.D, cfg.seed, stream=200 + n)
        oracle_layer(wl.pool, L0, cfg.k, u16(x), n_threads=ncores)
        n += 1
        if time.time() - t0 >= seconds:
            break
    dt = time.time() - t0
    t1 = time.time()
    oracle_layer(wl.pool, L0, cfg.k, u16(synth.hidden(1, cfg.D, cfg.seed, stream=299)), n_threads=1)
    dt1 = time.time() - t1
    extra = "" if sample_T == T else f"; a {sample_T}-token sample of the {T}-token batch, per-layer rate extrapolated"
    return {"value": round(n * sample_T / dt, 3), "unit": "tokens/s", "cores": ncores, "kind": "oracle",
            "sample": f"{n} steps of {sample_T} tokens (1 layer, full expert pass incl. routing), {dt:.1f} s{extra}",
            "single_thread": {"value": round(1.0 / dt1, 3), "unit": "tokens/s", "cores": 1,
                              "sample": "1 token, 1 layer"}}


def cpu_baseline_chain(cfg, wl):
    """The oracle on the host cores: decode48 — one token through all 48 layers;
    prefill48 — a 64-token sample through one layer (per-layer rate)."""
    from tests.harness import oracle_layer, u16
    ncores = os.cpu_count() or 1
    if cfg.T <= 8:
        x = u16(wl.x)
        t0 = time.time()
        for L in wl.layers:
            x = oracle_layer(wl.pool, L, cfg.k, x, residual_bits=x, n_threads=ncores).out
        dt = time.time() - t0
        return {"value": round(cfg.T * len(wl.layers) / dt, 3), "unit": "tokens/s (per layer)", "cores": ncores,
                "kind": "oracle", "sample": f"{cfg.T} token(s) through all {len(wl.layers)} layers, {dt:.1f} s"}
    xs = u16(wl.x[:64])
    t0 = time.time()
    oracle_layer(wl.pool, wl.layers[0], cfg.k, xs, residual_bits=xs, n_threads=ncores)
    dt = time.time() - t0
    return {"value": round(64 / dt, 3), "unit": "tokens/s (per layer)", "cores": ncores, "kind": "oracle",
            "sample": f"64 of the {cfg.T} tokens through layer 0, {dt:.1f} s; per-layer rate extrapolated"}


def run_reference(args, ws_, rank):
    """The oracle as it stands on the host cores: each step is the full expert
    pass (routing, slot lookup, every selected expert, combine) of one token of
    the headline workload; its 11 expert evaluations run in parallel over the
    cores."""
    if rank != 0:
        return
    cfg = _cfg("decode", args)
    wl = configs.build(cfg, device="cpu", T=1)
    from tests.harness import oracle_layer, u16
    ncores = os.cpu_count() or 1
    L0 = wl.layers[0]
    for w in range(args.warmup):
        oracle_layer(wl.pool, L0, cfg.k, u16(synth.hidden(1, cfg.D, cfg.seed, stream=300 + w)), n_threads=ncores)
    t0 = time.time()
    for s in range(args.steps):
        oracle_layer(wl.pool, L0, cfg.k, u16(synth.hidden(1, cfg.D, cfg.seed, stream=400 + s)), n_threads=ncores)
    dt = time.time() - t0
    value = args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": ws_,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (CPU oracle)",
            "data": "synthetic", "config": {"workload": cfg.name, "sample": "1 token per step"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": ncores, "kind": "oracle",
                             "sample": f"{args.steps} steps x 1 token of {cfg.name}"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main
def run_ours(args, ws_, rank, local):
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cpu = rank == 0 and ws_ == 1 and not args.no_cpu_baseline
    only = args.only
    head_name = only or "decode"
    cfg = _cfg(head_name, args)
    K, W = args.steps, args.warmup
    with _nvtx(head_name):
        if cfg.layers == 1:
            head = bench_layer(head_name, K, W, ws_, dev, local, args, cpu)
        else:
            head = bench_chain(head_name, K, W, ws_, dev, local, args, cpu)
    gc.collect()
    torch.cuda.empty_cache()
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": ws_, "steps": K, "warmup": W,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"{synth.FMT_NAMES[cfg.fmt]} weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded generator; no trained weights)",
        "config": {"workload": head["workload"], "global_batch": cfg.T * ws_, "l2": head["l2"],
                   "parallelism": f"replicas x{ws_}"},
        "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "roofline": head["roofline"],
        "clocks": head["clocks"],
    }
    for key in ("hit_rate", "u_hit_mean", "step_alg_bytes", "chain_tokens_per_s", "expert_loads", "three_calls",
                "fp8_variant"):
        if key in head:
            line[key] = head[key]
    if "cpu_baseline" in head:
        line["cpu_baseline"] = head["cpu_baseline"]
    if not only and not args.no_extra:
        # the other workloads: fixed, small step counts (each is far above L2 or
        # rotates replicas); the decode chain at 48 layers x K steps
        plan = {"prefill": (max(8, min(K, 64)), 3), "decode48": (max(8, min(K, 64)), 3),
                "prefill48": (3, 1), "decode_coder": (max(8, min(K, 64)), 3),
                "prefill_coder": (max(8, min(K, 64)), 3)}
        for name in EXTRA:
            k_, w_ = plan[name]
            fn = bench_layer if configs.CONFIGS[name].layers == 1 else bench_chain
            # the Coder shape: no oracle timing of its own (the 512-expert lines carry it)
            with _nvtx(name):
                line[name] = fn(name, k_, max(w_, 1), ws_, dev, local, args, cpu and not name.endswith("_coder"))
            gc.collect()
            torch.cuda.empty_cache()
        with _nvtx("small_batches"):
            line["small_batches"] = bench_small_batches(ws_, dev, local, args)
        gc.collect()
        torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--only", default=None, choices=list(configs.CONFIGS),
                    help="time this one workload as the headline (no other workloads)")
    ap.add_argument("--no-extra", action="store_true", help="headline workload only")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--replicas", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--nvtx", action="store_true",
                    help="NVTX ranges around each workload and each timed region (ncu --nvtx-include)")
    ap.add_argument("--seed", type=int, default=None,
                    help="seed of every synthetic input (default: each workload's own, 0 except tiny)")
    args = ap.parse_args()
    global NVTX
    NVTX = args.nvtx
    ws_, rank, local = _dist()
    if args.impl == "reference":
        run_reference(args, ws_, rank)
        return
    if args.warmup < 3:
        args.warmup = 3
    if ws_ > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    try:
        run_ours(args, ws_, rank, local)
    finally:
        if ws_ > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
