"""GPU parity of the edges between and inside the two paths, against the CPU
oracle through the C ABI:

* the path crossovers: T = 5 is the smallest batch of the tensor-core router
  (the expert pass still takes its decode path), T = 9 the smallest batch of
  the prefill expert pass; their first rows match the decode path on the same
  tokens;
* one expert set takes every token (router weights zero, a strictly
  decreasing bias): expert groups of 300 rows span several 128-row tiles and
  two 256-token plan chunks, on both paths;
* the 2,048-token prefill chunk with a 320-of-512 slot table: ids of every
  token bit-exact against the oracle's router, the complete miss list
  against the oracle's slot lookup, outputs on a 64-token sample;
* a chain of three layers whose pools use the three block formats in turn
  (per-layer mixed precision), on the decode and the prefill path.

Bars: ids and miss lists bit-exact, gates within 1e-6 relative, outputs within
relative L2 1e-2 per token."""
import os

import numpy as np
import pytest
import torch

import oracle
from bit_expert_ffn_route_b200 import configs, moe, synth
from tests.harness import bf16_from_u16, oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu

TOL_OUT = 1e-2
TOL_GATE = 1e-6
NCPU = os.cpu_count() or 8


def _layer(wl, L, k, T):
    return moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, k, T)


def _check_full(wl, L, x, k, residual=None):
    T = x.shape[0]
    layer = _layer(wl, L, k, T)
    out = layer(x, residual=residual)
    torch.cuda.synchronize()
    ref = oracle_layer(wl.pool, L, k, u16(x), residual_bits=None if residual is None else u16(residual),
                       n_threads=NCPU)
    assert np.array_equal(layer.ids.cpu().numpy(), ref.ids)
    g = layer.gates.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - ref.gates) <= TOL_GATE * np.abs(ref.gates) + 1e-12)
    n = int(layer.miss_count.item())
    assert n == len(ref.miss_list)
    assert np.array_equal(layer.miss_list[:n].cpu().numpy(), ref.miss_list)
    err = rel_l2_per_token(u16(out), ref.out)
    assert err.max() <= TOL_OUT, err
    assert moe.moe_workspace_status(layer.ws) == moe.MOE_OK
    return layer, out, ref


@pytest.mark.parametrize("T", [5, 8, 9, 24, 25])
def test_crossover_batches_and_decode_rows(T):
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=T, layers=1)
    L = wl.layers[0]
    _, outT, _ = _check_full(wl, L, wl.x, wl.cfg.k)
    layer4 = _layer(wl, L, wl.cfg.k, 4)
    out4 = layer4(wl.x[:4].contiguous())
    torch.cuda.synchronize()
    assert rel_l2_per_token(u16(outT)[:4], u16(out4)).max() <= TOL_OUT


@pytest.mark.parametrize("T", [4, 300])
def test_one_expert_set_takes_every_token(T):
    cfg = configs.CONFIGS["decode"]
    wl = configs.build(cfg, device="cuda", T=T, layers=1)
    L = wl.layers[0]
    # logits = bias exactly (Wr = 0): every token ranks experts 0, 1, ..., in order
    L.Wr = torch.zeros_like(L.Wr)
    L.bias = (-torch.arange(cfg.E, dtype=torch.float32) / 64.0).cuda()
    L.slot_table = (torch.arange(cfg.E, dtype=torch.int32) % 320).cuda()   # all resident
    layer, out, ref = _check_full(wl, L, wl.x, cfg.k)
    assert np.array_equal(ref.ids, np.tile(np.arange(cfg.k, dtype=np.int32), (T, 1)))
    assert int(layer.miss_count.item()) == 0


def test_prefill_2048_all_ids_and_full_miss_list():
    base = configs.CONFIGS["prefill"]
    cfg = configs.Config("prefill_320", 1, base.D, base.F, base.E, base.k, base.T, base.fmt, [320],
                         base.zipf_s, base.zipf_alpha)
    wl = configs.build(cfg, device="cuda")
    L = wl.layers[0]
    layer = _layer(wl, L, cfg.k, cfg.T)
    out = layer(wl.x)
    torch.cuda.synchronize()
    xb = u16(wl.x)
    table = L.slot_table.cpu().numpy()
    want_ids, want_g = oracle.topk_gates(oracle.router_logits(xb, u16(L.Wr), L.bias.cpu().numpy()), cfg.k)
    assert np.array_equal(layer.ids.cpu().numpy(), want_ids)
    g = layer.gates.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - want_g) <= TOL_GATE * np.abs(want_g) + 1e-12)
    _, want_miss = oracle.slot_lookup(want_ids, table, wl.pool.n_slots)
    n = int(layer.miss_count.item())
    assert n == len(want_miss) and n > 0
    assert np.array_equal(layer.miss_list[:n].cpu().numpy(), want_miss)
    sample = np.sort(np.random.default_rng(1).choice(cfg.T, 64, replace=False))
    ref = oracle_layer(wl.pool, L, cfg.k, xb[sample], n_threads=NCPU)
    assert rel_l2_per_token(u16(out)[sample], ref.out).max() <= TOL_OUT
    assert moe.moe_workspace_status(layer.ws) == moe.MOE_OK


@pytest.mark.parametrize("T", [4, 48])
def test_mixed_format_layer_chain(T):
    """Layers 0, 1, 2 use Q2_32, Q3_32 and Q3_S256 pools; each GPU layer runs on
    the oracle's input of that layer (values flow oracle -> GPU only)."""
    base = configs.CONFIGS["decode"]
    x_bits = u16(synth.hidden(T, base.D, seed=21, device="cpu"))
    for l, fmt in enumerate((synth.Q2_32, synth.Q3_32, synth.Q3_S256)):
        cfg = configs.Config(f"mixed{l}", 1, base.D, base.F, base.E, base.k, T, fmt, [320], 1.1, 0.47,
                             seed=30 + l, weight_std=0.008)
        wl = configs.build(cfg, device="cuda")
        L = wl.layers[0]
        x = bf16_from_u16(x_bits)
        layer = _layer(wl, L, cfg.k, T)
        out = layer(x, residual=x)
        torch.cuda.synchronize()
        ref = oracle_layer(wl.pool, L, cfg.k, x_bits, residual_bits=x_bits, n_threads=NCPU)
        assert np.array_equal(layer.ids.cpu().numpy(), ref.ids), l
        n = int(layer.miss_count.item())
        assert np.array_equal(layer.miss_list[:n].cpu().numpy(), ref.miss_list), l
        assert rel_l2_per_token(u16(out), ref.out).max() <= TOL_OUT, l
        x_bits = ref.out
