"""GPU side of the expert-cache calls (include/moe_cache.h), through the C ABI:
the popularity count against numpy's bincount, the slot copy bit-exact
through the oracle's dequantiser, and a decode layer that uses an expert
admitted by a plan (its weights copied into the slot of an evicted expert,
the slot table updated) against the oracle reading the same pool."""
import numpy as np
import pytest
import torch

import oracle
from bit_expert_ffn_route_b200 import configs, moe, synth
from tests.harness import mini_pool, oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu

TOL_OUT = 1e-2


def test_hist_matches_bincount_and_accumulates():
    rng = np.random.default_rng(3)
    T, k, E = 64, 10, 512
    ids = rng.integers(-3, E + 5, size=(T, k)).astype(np.int32)
    counts = torch.zeros(E, dtype=torch.int32, device="cuda")
    d_ids = torch.from_numpy(ids).cuda()
    moe.moe_expert_hist(d_ids, E, counts)
    moe.moe_expert_hist(d_ids, E, counts)
    torch.cuda.synchronize()
    v = ids[(ids >= 0) & (ids < E)]
    assert np.array_equal(counts.cpu().numpy(), 2 * np.bincount(v, minlength=E))


@pytest.mark.parametrize("fmt", [synth.Q2_32, synth.Q3_S256])
def test_slot_fill_bit_exact(fmt):
    D, F = 512, 256
    pool = synth.make_pool(fmt, D, F, 4, seed=5, device="cuda")
    P = moe.make_pool(pool, 0)
    before = [pool.slot_host(s) for s in range(4)]
    src = synth.make_pool(fmt, D, F, 1, seed=9, device="cpu", pool_id=3)
    hc = src.codes[:synth.slot_code_bytes(fmt, D, F)].clone().pin_memory()
    hs = src.scales[:synth.slot_scale_bytes(fmt, D, F)].clone().pin_memory()
    stream = torch.cuda.Stream()
    moe.moe_slot_fill(P, 2, hc, hs, stream=stream)
    stream.synchronize()
    hp, remap = mini_pool(src, [0], 0)
    for m in range(3):
        rows, K = (F, D) if m < 2 else (D, F)
        out = torch.empty(rows, K, dtype=torch.float32, device="cuda")
        moe.moe_dequantize(P, 2, m, out)
        torch.cuda.synchronize()
        want = oracle.dequant(hp, remap[0], m)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))
    # the other slots are untouched
    for s in (0, 1, 3):
        c1, s1 = pool.slot_host(s)
        assert np.array_equal(before[s][0], c1) and np.array_equal(before[s][1], s1)


def test_decode_uses_an_admitted_expert():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=4, layers=1)
    cfg, L = wl.cfg, wl.layers[0]
    x = wl.x
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, cfg.k, x.shape[0])
    layer(x)
    torch.cuda.synchronize()
    ids = layer.ids.cpu().numpy()
    table = L.slot_table.cpu().numpy()
    misses = [int(e) for e in np.unique(ids) if table[e] < 0]
    assert misses, "the workload has misses"
    # popularity from this batch: count through the kernel, then plan with the
    # slot table restricted to residents nobody selected (they are the weakest)
    counts = torch.zeros(cfg.E, dtype=torch.int32, device="cuda")
    moe.moe_expert_hist(layer.ids, cfg.E, counts)
    torch.cuda.synchronize()
    score = counts.cpu().numpy().astype(np.float32)
    slots = np.array(sorted(int(s) for s in table[table >= 0]), np.int32)
    moves, new_table = moe.moe_cache_plan(score, table, slots, hysteresis=1.0, max_moves=1)
    assert len(moves) == 1
    slot, evict, admit = (int(v) for v in moves[0])
    assert admit in misses and evict >= 0 and score[evict] == 0
    # the admitted expert's weights: a fresh expert in the pool's format
    src = synth.make_pool(wl.pool.fmt, cfg.D, cfg.F, 1, seed=11, device="cpu", pool_id=9)
    hc = src.codes[:synth.slot_code_bytes(wl.pool.fmt, cfg.D, cfg.F)].clone().pin_memory()
    hs = src.scales[:synth.slot_scale_bytes(wl.pool.fmt, cfg.D, cfg.F)].clone().pin_memory()
    copy = torch.cuda.Stream()
    copy.wait_stream(torch.cuda.current_stream())
    L.slot_table[evict] = -1                         # the evicted expert misses from here on
    moe.moe_slot_fill(moe.make_pool(wl.pool, L.shared_slot), slot, hc, hs, stream=copy)
    torch.cuda.current_stream().wait_stream(copy)
    L.slot_table.copy_(torch.from_numpy(new_table).cuda())
    layer2 = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, cfg.k, x.shape[0])
    out = layer2(x)
    torch.cuda.synchronize()
    assert int(layer2.miss_count.item()) < int(layer.miss_count.item())
    ref = oracle_layer(wl.pool, L, cfg.k, u16(x))
    assert np.array_equal(layer2.ids.cpu().numpy(), ref.ids)
    n = int(layer2.miss_count.item())
    assert np.array_equal(layer2.miss_list[:n].cpu().numpy(), ref.miss_list)
    err = rel_l2_per_token(u16(out), ref.out)
    assert err.max() <= TOL_OUT, err
