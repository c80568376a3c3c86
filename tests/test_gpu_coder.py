"""GPU parity of the 256-expert "Coder" shape (256 of the 512 routed experts
kept per layer; greenbean-ai "Strata 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next"
§四) against the CPU oracle, through the C ABI: the decode layer (one call and
three calls) and the 2,048-token prefill chunk.  Bars as for the 512-expert
workloads: ids and miss lists bit-exact, gates within 1e-6 relative, outputs
within relative L2 1e-2 per token."""
import numpy as np
import pytest
import torch

import oracle
from bit_expert_ffn_route_b200 import configs, moe
from tests.harness import oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu

TOL_OUT = 1e-2
TOL_GATE = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    moe.lib()


def _check_ids_gates(layer, ref_ids, ref_gates, idx):
    assert np.array_equal(layer.ids.cpu().numpy()[idx], ref_ids)
    g = layer.gates.cpu().numpy()[idx].astype(np.float64)
    assert np.all(np.abs(g - ref_gates) <= TOL_GATE * np.abs(ref_gates) + 1e-12)


@pytest.mark.parametrize("one_call", [False, True])
def test_coder_decode_parity(one_call):
    cfg = configs.CONFIGS["decode_coder"]
    wl = configs.build(cfg, device="cuda", layers=1)
    L = wl.layers[0]
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, cfg.k, cfg.T)
    out = layer.fused(wl.x) if one_call else layer(wl.x, with_logits=True)
    torch.cuda.synchronize()
    ref = oracle_layer(wl.pool, L, cfg.k, u16(wl.x))
    if not one_call:                 # the CUDA-core router returns the canonical logits themselves
        assert np.array_equal(layer.logits.cpu().numpy().view(np.uint32), ref.logits.view(np.uint32))
    _check_ids_gates(layer, ref.ids, ref.gates, np.arange(cfg.T))
    assert int(layer.miss_count.item()) == 0 == len(ref.miss_list)
    assert ref.ids.max() < 256
    err = rel_l2_per_token(u16(out), ref.out)
    assert err.max() <= TOL_OUT, err


def test_coder_prefill_2048_tokens():
    """Every token's ids and gates against the oracle's router; outputs on a
    64-token sample (the oracle's expert pass at 2,048 tokens takes minutes)."""
    cfg = configs.CONFIGS["prefill_coder"]
    wl = configs.build(cfg, device="cuda")
    L = wl.layers[0]
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, cfg.k, cfg.T)
    out = layer(wl.x)
    torch.cuda.synchronize()
    logits = oracle.router_logits(u16(wl.x), u16(L.Wr), L.bias.cpu().numpy())
    ref_ids, ref_gates = oracle.topk_gates(logits, cfg.k)
    _check_ids_gates(layer, ref_ids, ref_gates, np.arange(cfg.T))
    assert int(layer.miss_count.item()) == 0
    assert int(layer.ws[4:8].view(torch.int32).item()) == 0     # device error word
    sample = np.sort(np.random.default_rng(1).choice(cfg.T, 64, replace=False))
    ref = oracle_layer(wl.pool, L, cfg.k, u16(wl.x)[sample], n_threads=16)
    assert np.array_equal(ref.ids, ref_ids[sample])
    err = rel_l2_per_token(u16(out)[sample], ref.out)
    assert err.max() <= TOL_OUT, err
    loads = np.bincount(ref_ids.ravel(), minlength=cfg.E)
    assert loads.max() >= 200
