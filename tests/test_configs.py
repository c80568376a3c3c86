"""The synthetic workloads are well formed (CPU only): every layer's slot table
maps exactly its resident experts to distinct slots of the pool, the shared
experts sit in slots of their own, the bias follows the recipe, and a seed
reproduces the same workload bit for bit."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_route_b200 import configs, synth


def _no_weights(fmt, D, F, n_slots, seed, device="cpu", **kw):
    """A pool of the right slot count without generated weights (the structure
    checks need none; the full pools run to gigabytes)."""
    e = torch.empty(0, dtype=torch.uint8)
    return synth.PoolData(fmt, D, F, n_slots, e, e, 0, 0)


@pytest.mark.parametrize("name", configs.ORDER)
def test_workload_structure(name, monkeypatch):
    cfg = configs.CONFIGS[name]
    L = min(cfg.layers, 2)
    monkeypatch.setattr(configs.synth, "make_pool", _no_weights)
    wl = configs.build(cfg, T=4, layers=L)
    assert len(wl.layers) == L
    n_slots = wl.pool.n_slots
    want = [cfg.E] * L if cfg.resident_per_layer is None else list(cfg.resident_per_layer[:L])
    assert n_slots == sum(want) + L
    used = []
    for l, lay in enumerate(wl.layers):
        st = lay.slot_table.numpy()
        assert lay.slot_table.dtype == torch.int32 and st.shape == (cfg.E,)
        res = st[st >= 0]
        assert len(res) == want[l]
        assert np.all(st[st < 0] == -1)
        used += res.tolist() + [lay.shared_slot]
        assert lay.Wr.shape == (cfg.E, cfg.D) and lay.Wr.dtype == torch.bfloat16
        assert (lay.bias is None) == (cfg.zipf_s is None)
        if cfg.resident_per_layer is not None:
            # the resident experts are the layer's most popular ones
            order = synth.popularity_order(cfg.E, cfg.seed, l).numpy()
            assert set(np.nonzero(st >= 0)[0].tolist()) == set(order[:want[l]].tolist())
    assert len(set(used)) == len(used) == n_slots            # every slot used once
    assert min(used) == 0 and max(used) == n_slots - 1
    assert wl.x.shape == (4, cfg.D) and wl.x.dtype == torch.bfloat16


def test_bias_is_the_zipf_recipe():
    cfg = configs.CONFIGS["decode"]
    b = synth.zipf_bias(cfg.E, cfg.zipf_s, cfg.zipf_alpha, cfg.seed, 0).double().numpy()
    order = synth.popularity_order(cfg.E, cfg.seed, 0).numpy()
    ranks = np.arange(1, cfg.E + 1)
    want = (-cfg.zipf_alpha * cfg.zipf_s * np.log(ranks)).astype(np.float32)
    assert np.array_equal(b[order].astype(np.float32), want)
    assert np.all(np.diff(b[order]) <= 0)                     # more popular, larger bias


def test_seed_reproduces_the_workload():
    cfg = configs.CONFIGS["tiny"]
    a, b = configs.build(cfg), configs.build(cfg)
    assert torch.equal(a.pool.codes, b.pool.codes) and torch.equal(a.pool.scales, b.pool.scales)
    assert torch.equal(a.x.view(torch.int16), b.x.view(torch.int16))
    assert torch.equal(a.layers[0].Wr.view(torch.int16), b.layers[0].Wr.view(torch.int16))
    import dataclasses
    c = configs.build(dataclasses.replace(cfg, seed=cfg.seed + 1))
    assert not torch.equal(a.pool.codes, c.pool.codes)
    assert not torch.equal(a.x.view(torch.int16), c.x.view(torch.int16))
