"""Large-prefill workload on one GPU: 4,096 tokens x 48 layers, Q3_S256
super-blocks, every one of the 512 experts of every layer resident (~50 GB of
expert weights in HBM), uniform routing, residual chain.

The oracle carries 64 sampled tokens through all 48 layers on its own.  At
each layer the GPU runs the full 4,096-token batch, whose 64 sample rows are
set to the oracle's input of that layer (values flow oracle -> GPU only; the
other rows carry the GPU's own chain).  On the sample rows: ids bit-exact,
gates within 1e-6 relative, no misses, outputs within relative L2 1e-2 per
token."""
import os

import numpy as np
import pytest
import torch

from bit_expert_ffn_route_b200 import configs, moe
from tests.harness import bf16_from_u16, oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu

TOL_OUT = 1e-2
TOL_GATE = 1e-6


def test_prefill48_per_layer_on_sample():
    cfg = configs.CONFIGS["prefill48"]
    wl = configs.build(cfg, device="cuda")
    assert wl.pool.n_slots == 48 * 513
    sample = torch.from_numpy(np.sort(np.random.default_rng(4).choice(cfg.T, 64, replace=False))).cuda()
    x_gpu = wl.x
    x_or = u16(wl.x[sample])
    worst = 0.0
    layers = {}
    for l, L in enumerate(wl.layers):
        x_in = x_gpu.clone()
        x_in[sample] = bf16_from_u16(x_or)
        layer = layers.setdefault(0, moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, cfg.k, cfg.T))
        layer.pool = moe.make_pool(wl.pool, L.shared_slot)
        layer.slot_table, layer.Wr, layer.bias = L.slot_table, L.Wr, L.bias
        out = layer(x_in, residual=x_in, out=torch.empty_like(x_in))
        torch.cuda.synchronize()
        ref = oracle_layer(wl.pool, L, cfg.k, x_or, residual_bits=x_or, n_threads=os.cpu_count() or 8)
        idx = sample.cpu().numpy()
        assert np.array_equal(layer.ids.cpu().numpy()[idx], ref.ids), l
        g = layer.gates.cpu().numpy()[idx].astype(np.float64)
        assert np.all(np.abs(g - ref.gates) <= TOL_GATE * np.abs(ref.gates) + 1e-12), l
        assert int(layer.miss_count.item()) == 0 and len(ref.miss_list) == 0
        err = rel_l2_per_token(u16(out)[idx], ref.out)
        worst = max(worst, float(err.max()))
        assert err.max() <= TOL_OUT, (l, err.max())
        assert moe.moe_workspace_status(layer.ws) == moe.MOE_OK, l
        x_gpu = out
        x_or = ref.out
    print(f"prefill48: worst rel L2 over 48 layers x 64 tokens {worst:.2e}")
    del wl, layers
    torch.cuda.empty_cache()
