"""Host-side helpers of bench.py (CPU only): the DRAM-traffic records are looked
up by workload name and reported only while the kernels' sources are the
captured ones; --seed replaces every workload's seed and nothing else; the
per-launch percentiles; --nvtx ranges, off unless asked for and balanced."""
import argparse
import hashlib
import json
import os

import numpy as np

import bench
from bit_expert_ffn_route_b200 import configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_records_are_per_workload():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        records = json.load(f)
    for name, rec in records.items():
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        assert os.path.exists(os.path.join(ROOT, rec["profile"])), rec["profile"]
        # the figure is reported only while the kernel's sources are the captured ones
        want = (rec["bytes_per_launch"], rec["covers"]) if h.hexdigest() == rec["sha256"] else (None, None)
        assert bench._traffic(name) == want
    # every record belongs to a bench workload (or its e4m3 variant)
    for name in records:
        assert name.removesuffix("_fp8") in configs.CONFIGS, name
    # a workload without a capture of its own gets no traffic figure
    assert bench._traffic("decode48") == (None, None)
    assert bench._traffic("decode_three_calls") == (None, None)


def test_seed_option_replaces_only_the_seed():
    for name, cfg in configs.CONFIGS.items():
        assert bench._cfg(name, argparse.Namespace(seed=None)) is cfg
        other = bench._cfg(name, argparse.Namespace(seed=7))
        assert other.seed == 7
        assert {**vars(other), "seed": cfg.seed} == vars(cfg)


def test_percentiles_in_microseconds():
    ms = np.linspace(0.010, 0.020, 101)           # 10 .. 20 us
    assert bench._pct_us(ms) == [11.0, 15.0, 19.0]


def test_nvtx_ranges_are_opt_in_and_balanced():
    calls = []
    push, pop = bench.torch.cuda.nvtx.range_push, bench.torch.cuda.nvtx.range_pop
    try:
        bench.torch.cuda.nvtx.range_push = lambda name: calls.append(("push", name))
        bench.torch.cuda.nvtx.range_pop = lambda: calls.append(("pop",))
        with bench._nvtx("off"):
            pass
        assert calls == []
        bench.NVTX = True
        try:
            with bench._nvtx("workload"):
                with bench._nvtx("timed"):
                    raise KeyError("inside")
        except KeyError:
            pass
        assert calls == [("push", "workload"), ("push", "timed"), ("pop",), ("pop",)]
    finally:
        bench.NVTX = False
        bench.torch.cuda.nvtx.range_push, bench.torch.cuda.nvtx.range_pop = push, pop
