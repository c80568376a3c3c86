"""GPU parity of the prefill path (T > 24: permute + tcgen05 grouped GEMMs)
against the CPU oracle, through the C ABI.  Bars as for the decode path:
routing ids and miss lists bit-exact; outputs within relative L2 1e-2 per token
(fp16 tensor-core operands and bf16 y rows on this path, fp32 accumulation)."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_route_b200 import configs, moe, synth
import oracle
from tests.harness import f64, oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu

TOL_OUT = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    moe.lib()


def _run(wl, x, k=None, residual=None):
    k = k or wl.cfg.k
    L = wl.layers[0]
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, k, x.shape[0])
    out = layer(x, residual=residual)
    torch.cuda.synchronize()
    return layer, out


def _check(wl, x, sample=None, residual=None):
    layer, out = _run(wl, x, residual=residual)
    L = wl.layers[0]
    idx = np.arange(x.shape[0]) if sample is None else np.asarray(sample)
    xs = u16(x)[idx]
    ref = oracle_layer(wl.pool, L, wl.cfg.k, xs, residual_bits=None if residual is None else u16(residual)[idx],
                       n_threads=16)
    assert np.array_equal(layer.ids.cpu().numpy()[idx], ref.ids)
    g = layer.gates.cpu().numpy()[idx].astype(np.float64)
    assert np.all(np.abs(g - ref.gates) <= 1e-6 * np.abs(ref.gates) + 1e-12)
    assert int(layer.ws[4:8].view(torch.int32).item()) == 0     # device error word
    assert int(layer.route_ws[4:8].view(torch.int32).item()) == 0
    err = rel_l2_per_token(u16(out)[idx], ref.out)
    assert err.max() <= TOL_OUT, err
    if sample is None:
        n = int(layer.miss_count.item())
        assert n == len(ref.miss_list)
        assert np.array_equal(layer.miss_list[:n].cpu().numpy(), ref.miss_list)
    return layer, out, err


def test_prefill_tiny_64_tokens():
    wl = configs.build(configs.CONFIGS["tiny"], device="cuda", T=64)
    _check(wl, wl.x)


def test_prefill_decode_shapes_with_misses():
    # decode-layer shapes (320/512 resident) through the prefill path
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=40)
    layer, out, err = _check(wl, wl.x)
    assert int(layer.miss_count.item()) > 0


def test_prefill_matches_decode_path():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=32)
    _, out32 = _run(wl, wl.x)
    _, out4 = _run(wl, wl.x[:4].contiguous())
    err = rel_l2_per_token(u16(out32)[:4], u16(out4))
    assert err.max() <= TOL_OUT, err


@pytest.mark.parametrize("fmt", [synth.Q3_32, synth.Q3_S256])
def test_prefill_other_formats(fmt):
    base = configs.CONFIGS["decode"]
    cfg = configs.Config("pf", 1, base.D, base.F, base.E, base.k, 48, fmt, None, None, None)
    wl = configs.build(cfg, device="cuda")
    _check(wl, wl.x)


def test_prefill_residual_and_determinism():
    wl = configs.build(configs.CONFIGS["tiny"], device="cuda", T=96)
    res = synth.hidden(96, wl.cfg.D, seed=5, device="cuda")
    layer, out, _ = _check(wl, wl.x, residual=res)
    a = out.clone()
    b = layer(wl.x, residual=res)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.uint16), b.view(torch.uint16))


def test_prefill_config_2048_tokens():
    """Prefill-chunk workload: 2,048 tokens, Zipf(0.8)-skewed expert loads,
    every expert resident.  Outputs checked on a 64-token sample."""
    cfg = configs.CONFIGS["prefill"]
    wl = configs.build(cfg, device="cuda")
    g = np.random.default_rng(0)
    sample = np.sort(g.choice(cfg.T, 64, replace=False))
    layer, out, err = _check(wl, wl.x, sample=sample)
    assert int(layer.miss_count.item()) == 0
    ids = layer.ids.cpu().numpy()
    loads = np.bincount(ids.ravel(), minlength=cfg.E)
    print(f"prefill loads: max {loads.max()}, zero-load experts {(loads == 0).sum()}, worst rel L2 {err.max():.2e}")
    assert loads.max() >= 200


def test_prefill_router_logits_bound_and_canonical_selection():
    """Prefill router: tensor-core logits within 2^-12 |x|_2 |Wr_e|_2 of the
    canonical ones; ids and gates from the canonical logits of the candidates,
    so they match the oracle exactly (ids) / within 1e-6 (gates)."""
    cfg = configs.CONFIGS["prefill"]
    wl = configs.build(cfg, device="cuda", T=192)
    L = wl.layers[0]
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, cfg.k, 192)
    moe.moe_route_topk(wl.x, L.Wr, L.bias, cfg.k, layer.ids, layer.gates, layer.route_ws, logits=layer.logits)
    torch.cuda.synchronize()
    xb, wb = u16(wl.x), u16(L.Wr)
    ref_l = oracle.router_logits(xb, wb, L.bias.cpu().numpy())
    ref_ids, ref_g = oracle.topk_gates(ref_l, cfg.k)
    assert np.array_equal(layer.ids.cpu().numpy(), ref_ids)
    g = layer.gates.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - ref_g) <= 1e-6 * np.abs(ref_g) + 1e-12)
    xn = np.linalg.norm(f64(xb), axis=1)
    wn = np.linalg.norm(f64(wb), axis=1)
    bound = 2.0 ** -12 * np.outer(xn, wn)
    dev = np.abs(layer.logits.cpu().numpy().astype(np.float64) - ref_l.astype(np.float64))
    assert np.all(dev <= bound), float((dev / bound).max())
    assert int(layer.route_ws[4:8].view(torch.int32).item()) == 0
