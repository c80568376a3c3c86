"""The device error word of a workspace, shown without any GPU fault.

A bounded device wait is made to run out on a device flag that nothing sets
(a one-thread test kernel with a 20 ms limit).  The wait sets the timeout bit,
moe_workspace_status reports MOE_ERR_TIMEOUT, an expert pass on that
workspace then does no work (it gives up at once), and after the caller
re-zeroes the workspace header the same pass matches the oracle again."""
import time

import numpy as np
import pytest
import torch

from bit_expert_ffn_route_b200 import configs, moe
from tests.harness import oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu


def test_wait_runs_out_sets_timeout():
    ws = moe.alloc_ws(1024)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    t0 = time.time()
    moe.moe_debug_wait_flag(flag, 1, 20000, ws)          # nothing ever sets the flag
    assert moe.moe_workspace_status(ws) == moe.MOE_ERR_TIMEOUT
    assert time.time() - t0 < 5.0
    # a satisfied wait leaves a clean word clean
    ws2 = moe.alloc_ws(1024)
    flag.fill_(1)
    moe.moe_debug_wait_flag(flag, 1, 20000, ws2)
    assert moe.moe_workspace_status(ws2) == moe.MOE_OK


def test_timeout_bit_stops_later_calls_until_cleared():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", layers=1)
    L = wl.layers[0]
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 4)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_debug_wait_flag(flag, 1, 10000, layer.ws)   # expert-pass workspace: timeout bit set
    layer.expert_out.fill_(0)
    layer.miss_count.fill_(-7)
    t0 = time.time()
    layer(wl.x)
    torch.cuda.synchronize()
    assert time.time() - t0 < 0.4                          # well under one 500 ms wait limit
    assert moe.moe_workspace_status(layer.ws) == moe.MOE_ERR_TIMEOUT
    assert int(layer.miss_count.item()) == -7              # the expert pass did no work
    assert int(layer.expert_out.count_nonzero().item()) == 0
    # router workspace: a preset timeout bit makes the router write ids -1, gates 0
    moe.moe_debug_wait_flag(flag, 1, 10000, layer.route_ws)
    layer(wl.x)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(layer.route_ws) == moe.MOE_ERR_TIMEOUT
    assert bool((layer.ids == -1).all()) and bool((layer.gates == 0).all())
    # the caller clears both headers: the next call is correct again
    layer.ws[:1024].zero_()
    layer.route_ws[:8].zero_()
    out = layer(wl.x)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(layer.ws) == moe.MOE_OK
    assert moe.moe_workspace_status(layer.route_ws) == moe.MOE_OK
    ref = oracle_layer(wl.pool, L, wl.cfg.k, u16(wl.x))
    assert np.array_equal(layer.ids.cpu().numpy(), ref.ids)
    assert rel_l2_per_token(u16(out), ref.out).max() <= 1e-2
