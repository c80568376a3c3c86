"""The synthetic workloads have the routing structure the pages report, as the
oracle's router computes it from the generated inputs (CPU only):

- decode (320 of 512 experts resident, Zipf(1.1) popularity bias): the share
  of (token, rank) pairs whose expert is resident is near the 93.4% GPU
  expert-cache hit rate of the wiselychen RTX 5090 report §2;
- prefill chunk (2,048 tokens, Zipf(0.8) bias): expert loads are skewed — some
  experts get hundreds of tokens, some none — and every token's k experts
  are distinct."""
import numpy as np

import oracle
from bit_expert_ffn_route_b200 import configs, synth
from tests.harness import u16


def _route(cfg, T, x_stream=0):
    Wr = synth.router_weight(cfg.E, cfg.D, cfg.seed, 0)
    bias = synth.zipf_bias(cfg.E, cfg.zipf_s, cfg.zipf_alpha, cfg.seed, 0).numpy()
    x = synth.hidden(T, cfg.D, cfg.seed, stream=x_stream)
    logits = oracle.router_logits(u16(x), u16(Wr), bias)
    return oracle.topk_gates(logits, cfg.k)


def test_decode_hit_rate_near_the_reported_cache_hit_rate():
    cfg = configs.CONFIGS["decode"]
    ids, _ = _route(cfg, 256, x_stream=7)             # 64 batches of 4 tokens
    resident = synth.popularity_order(cfg.E, cfg.seed, 0)[:cfg.resident_per_layer[0]].numpy()
    hit = np.isin(ids, resident).mean()
    assert 0.88 <= hit <= 0.98, hit


def test_prefill_loads_are_skewed():
    cfg = configs.CONFIGS["prefill"]
    ids, gates = _route(cfg, cfg.T)
    assert all(len(set(row)) == cfg.k for row in ids.tolist())
    load = np.bincount(ids.ravel(), minlength=cfg.E)
    assert load.sum() == cfg.T * cfg.k
    assert load.max() >= 200 and (load == 0).any(), (load.max(), (load == 0).sum())
    top = np.sort(load)[::-1]
    assert top[: cfg.E // 10].sum() > 0.5 * load.sum()    # a tenth of the experts take over half the rows
    assert np.allclose(gates.sum(axis=1), 1.0, atol=1e-12)


def test_coder_shape_routes_over_256_experts():
    """The Coder shape keeps 256 of the 512 routed experts: every id is below
    256, and the 2,048-token chunk's loads stay skewed under the same bias."""
    cfg = configs.CONFIGS["prefill_coder"]
    assert cfg.E == 256 and configs.CONFIGS["decode_coder"].E == 256
    ids, gates = _route(cfg, cfg.T)
    assert ids.min() >= 0 and ids.max() < 256
    assert all(len(set(row)) == cfg.k for row in ids.tolist())
    load = np.bincount(ids.ravel(), minlength=cfg.E)
    assert load.max() >= 200
    assert np.allclose(gates.sum(axis=1), 1.0, atol=1e-12)
