"""Benchmark of the routed-MoE expert pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode] [--impl ours|reference]

A step is one pass of the whole hot path — router logits + top-k + gates,
slot lookup + miss list, expert FFNs, combine — over one batch of synthetic
tokens at the workload's shapes.  Prints one JSON line (rank 0).

Timing: CUDA graphs of up to 512 steps are replayed until exactly K steps ran;
barrier + synchronize on both sides; CUDA events on the launching stream; max
over ranks.  L2 is defeated by rotating over R replicas of the expert pool,
router weights and token batches (R * per-step bytes >> 126 MB L2).
Per-kernel durations come from external event nodes inside the same graph.
"""
from __future__ import annotations

import argparse
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


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _traffic(kind):
    """DRAM bytes per launch from the committed ncu capture of this kernel, or
    None when the kernel's sources changed since the counters were taken."""
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


def run_ours(args, ws_, rank, local):
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = configs.CONFIGS[args.config]
    if cfg.layers != 1:
        raise SystemExit(f"bench.py times single-layer workloads; {cfg.name} is a parity case")
    T, D, F, E, k = cfg.T, cfg.D, cfg.F, cfg.E, cfg.k
    wl = configs.build(cfg, device=dev)
    L0 = wl.layers[0]
    slot_bytes = wl.pool.slot_bytes
    pool_bytes = wl.pool.n_slots * slot_bytes
    # decode touches ~(U+1) experts + Wr (~50 MB) per step: 8 replicas put ~350 MB
    # of other traffic between two uses of one replica (L2 is 126 MB)
    R = args.replicas or (8 if T <= 4 else 2)
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
    # per batch: distinct resident experts hit (deterministic per batch)
    table = L0.slot_table.cpu().numpy()
    u_hit, hits = [], []
    with torch.cuda.stream(stream):
        for r in range(R):
            layers[r](xs[r])
    torch.cuda.synchronize()
    for r in range(R):
        ids = layers[r].ids.cpu().numpy()
        sl = table[ids]
        u_hit.append(len(np.unique(sl[sl >= 0])))
        hits.append(float((sl >= 0).mean()))
    x_bytes = T * D * 2
    wr_bytes = E * D * 2
    fwd_bytes = [(u + 1) * slot_bytes + x_bytes for u in u_hit]         # expert weights read + x
    step_bytes = [fb + wr_bytes + x_bytes for fb in fwd_bytes]           # + router weights + out
    # algorithmic FLOPs of the expert FFNs: every resident (token, rank) row and
    # every token's shared-expert row costs gate + up + down = 3 * 2 * D * F
    fwd_flops = [(h * T * k + T) * 6.0 * D * F for h in hits]

    K, W = args.steps, args.warmup
    G = _divisor_at_most(K, 512)
    ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(G)]

    def step(i, timed=True):
        lay = layers[i % R]
        moe.moe_route_topk(xs[i % R], lay.Wr, lay.bias, k, lay.ids, lay.gates, lay.route_ws, stream=stream)
        if timed:
            ev[i][0].record(stream)
        moe.moe_expert_forward(lay.pool, lay.slot_table, xs[i % R], lay.ids, k, lay.expert_out, lay.miss_list,
                               lay.miss_count, lay.ws, stream=stream)
        if timed:
            ev[i][1].record(stream)
        moe.moe_combine(lay.expert_out, lay.gates, T, D, k, lay.out, stream=stream)

    graph = _graph_of(step, G, stream)
    # CUDAGraph.replay() launches on the current stream: replay on the timing stream
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-W // G))):
            graph.replay()
    torch.cuda.synchronize()
    if ws_ > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(K // G):
            graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    if ws_ > 1:
        torch.distributed.barrier()
    ms = t0.elapsed_time(t1)
    fwd_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(G)]
    ms = max_over_ranks(ms, ws_, dev)
    ms_per_step = ms / K
    value = ws_ * T * K / (ms / 1e3)
    hbm, tf, tf_sus, peak_kind = _peaks()
    fwd_avg_ms = float(np.mean(fwd_ms))
    fwd_alg = float(np.mean([fwd_bytes[i % R] for i in range(G)]))
    fwd_fl = float(np.mean([fwd_flops[i % R] for i in range(G)]))
    traffic, traffic_covers = _traffic("decode" if T <= 4 else "prefill")
    if T <= 4:
        achieved = fwd_alg / (fwd_avg_ms / 1e3) / 1e9
        roofline = {"kernel": "moe_expert_forward (decode_ffn_kernel: gate|up + down dequant-GEMV)", "bound": "hbm",
                    "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                    "traffic": traffic, "traffic_covers": traffic_covers, "peak_kind": f"{peak_kind} copy bandwidth",
                    "algorithmic_bytes_per_launch": round(fwd_alg), "avg_launch_us": round(fwd_avg_ms * 1e3, 3)}
    else:
        achieved = fwd_fl / (fwd_avg_ms / 1e3) / 1e12
        roofline = {"kernel": "moe_expert_forward (plan + tcgen05 gate|up and down grouped GEMMs)", "bound": "tensor",
                    "achieved": round(achieved, 1), "peak": tf_sus, "unit": "TFLOP/s", "frac": round(achieved / tf_sus, 4),
                    "traffic": traffic, "traffic_covers": traffic_covers, "peak_kind": f"{peak_kind} bf16 sustained (burst {tf})",
                    "algorithmic_flops_per_launch": round(fwd_fl), "avg_launch_us": round(fwd_avg_ms * 1e3, 3)}

    # end to end through the public API: pinned host input -> device, the three
    # calls, device -> pinned host output, every step
    xh = [torch.empty(T, D, dtype=torch.bfloat16).pin_memory() for _ in range(R)]
    oh = [torch.empty(T, D, dtype=torch.bfloat16).pin_memory() for _ in range(R)]
    for r in range(R):
        xh[r].copy_(xs[r].cpu())
    xd = [torch.empty(T, D, dtype=torch.bfloat16, device=dev) for _ in range(R)]

    def e2e_step(i):
        r = i % R
        xd[r].copy_(xh[r], non_blocking=True)
        lay = layers[r]
        lay(xd[r], stream=stream)
        oh[r].copy_(lay.out, non_blocking=True)

    Ke = K
    Ge = _divisor_at_most(Ke, 256)
    g2 = _graph_of(e2e_step, Ge, stream)
    with torch.cuda.stream(stream):
        g2.replay()
    torch.cuda.synchronize()
    if ws_ > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(Ke // Ge):
            g2.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ems = e0.elapsed_time(e1)
    ems = max_over_ranks(ems, ws_, dev)
    e2e_value = ws_ * T * Ke / (ems / 1e3)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws_, "steps": K, "warmup": W,
        "ms_per_step": round(ms_per_step, 6), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"{synth.FMT_NAMES[cfg.fmt]} weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded generator; no trained weights)",
        "config": {"workload": f"{cfg.name}: 1 layer, T={T}, D={D}, F={F}, E={E}, top-{k}+1 shared, "
                               f"{synth.FMT_NAMES[cfg.fmt]}, {int((table >= 0).sum())}/{E} resident",
                   "global_batch": T * ws_, "l2": f"rotating {R} replicas of pool+Wr+x ({R * pool_bytes / 1e9:.2f} GB)",
                   "parallelism": f"replicas x{ws_}"},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": T * D * 2,
                "d2h_bytes_per_step": T * D * 2},
        "gpu_launches": (3 if T <= 4 else 10) * K,
        "roofline": roofline,
        "hit_rate": round(float(np.mean(hits)), 4), "u_hit_mean": round(float(np.mean(u_hit)), 2),
        "step_alg_bytes": round(float(np.mean(step_bytes))),
        "clocks": clk.summary(),
    }
    if rank == 0 and ws_ == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, wl, seconds=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)


def cpu_baseline(cfg, wl, seconds=10.0):
    """The oracle as it stands, on this host's cores, on whole steps of the same workload."""
    import oracle
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
    return {"value": round(n * sample_T / dt, 3), "unit": "tokens/s", "cores": ncores, "kind": "oracle",
            "sample": f"{n} steps of {sample_T} tokens (1 layer, full expert pass incl. routing), {dt:.1f} s"}


def run_reference(args, ws_, rank):
    """The oracle as it stands on the host cores: each step is the full expert
    pass (routing, slot lookup, every selected expert, combine) of one token of
    the workload; its 11 expert evaluations run in parallel over the cores."""
    if rank != 0:
        return
    cfg = configs.CONFIGS[args.config]
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4096)
    ap.add_argument("--warmup", type=int, default=256)
    ap.add_argument("--config", default="decode", choices=list(configs.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--replicas", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    ws_, rank, local = _dist()
    if args.impl == "reference":
        run_reference(args, ws_, rank)
        return
    if args.warmup < 3:
        args.warmup = 3
    if ws_ > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        run_ours(args, ws_, rank, local)
    finally:
        if ws_ > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
