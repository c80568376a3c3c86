"""The multi-GPU bench path runs independent replicas (the pass does not
shard for the decode workload); its only cross-rank step is the timing: every
rank's elapsed time is reduced to the maximum, which every rank then uses.
Checked with two gloo ranks on CPU, as bench.py calls it."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        import bench
        dist.barrier()
        got = bench.max_over_ranks(10.0 + 3.5 * rank, ws, torch.device("cpu"))
        got2 = bench.max_over_ranks(-1.0 - rank, ws, torch.device("cpu"))
        out[rank] = (got, got2)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ws = 2
    with mp.get_context("spawn").Manager() as m:        # no fork of this (threaded) process
        out = m.dict()
        mp.start_processes(_rank, args=(ws, _free_port(), out), nprocs=ws, start_method="spawn")
        res = dict(out)
    assert res == {0: (13.5, -1.0), 1: (13.5, -1.0)}


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(4.25, 1, torch.device("cpu")) == 4.25
