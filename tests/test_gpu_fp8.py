"""GPU parity of the e4m3-operand expert pass (moe_expert_forward_fp8) through
the C ABI.  Against the oracle's definition of this variant (weights
e4m3(fp16(64 w)), x and h in e4m3, fp32 accumulation scaled by 1/64): ids and
miss lists bit-exact, outputs within relative L2 1e-2 per token, the bar of the
exact path.  Against the exact-weight oracle the e4m3 roundings cost accuracy:
the measured per-token error is asserted below TOL_VS_EXACT and printed."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_route_b200 import configs, moe, synth
from tests.harness import oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu

TOL_OUT = 1e-2          # GPU e4m3 path vs the oracle's e4m3 variant
# GPU e4m3 path vs the exact-weight oracle (the variant's loss).  e4m3 keeps 3
# mantissa bits: a rounding moves a value by up to 2^-4 of itself (RMS ~3.6%);
# x and the weights, then h, each take one, so y moves by several percent.
# Measured on the 2,048-token workload's 64-token sample: median 6.6e-2,
# p90 7.4e-2, max 8.2e-2.
TOL_VS_EXACT = 1e-1


@pytest.fixture(scope="module", autouse=True)
def _lib():
    moe.lib()


def _check(wl, x, sample=None, vs_exact=False):
    L = wl.layers[0]
    k = wl.cfg.k
    T = x.shape[0]
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, k, T)
    out = layer(x, fp8=True).clone()
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(layer.ws_fp8) == moe.MOE_OK
    idx = np.arange(T) if sample is None else np.asarray(sample)
    xs = u16(x)[idx]
    ref = oracle_layer(wl.pool, L, k, xs, n_threads=16, fp8=True)
    assert np.array_equal(layer.ids.cpu().numpy()[idx], ref.ids)
    err = rel_l2_per_token(u16(out)[idx], ref.out)
    assert err.max() <= TOL_OUT, err
    if sample is None:
        n = int(layer.miss_count.item())
        assert n == len(ref.miss_list)
        assert np.array_equal(layer.miss_list[:n].cpu().numpy(), ref.miss_list)
    loss = None
    if vs_exact:
        ex = oracle_layer(wl.pool, L, k, xs, n_threads=16)
        loss = rel_l2_per_token(u16(out)[idx], ex.out)
        print(f"e4m3 vs exact-weight oracle: median {np.median(loss):.3e}, p90 {np.quantile(loss, 0.9):.3e}, "
              f"max {loss.max():.3e}; vs its own definition max {err.max():.3e}")
        assert loss.max() <= TOL_VS_EXACT, loss
    return layer, out, err, loss


def test_fp8_prefill_2048_tokens():
    cfg = configs.CONFIGS["prefill"]
    wl = configs.build(cfg, device="cuda")
    sample = np.sort(np.random.default_rng(0).choice(cfg.T, 64, replace=False))
    layer, out, _, _ = _check(wl, wl.x, sample=sample, vs_exact=True)
    # the routing and the expert-pass row map are the exact path's
    ref = moe.Layer(wl.pool, wl.layers[0].shared_slot, wl.layers[0].slot_table, wl.layers[0].Wr, wl.layers[0].bias,
                    cfg.k, cfg.T)
    ref(wl.x)
    torch.cuda.synchronize()
    assert torch.equal(ref.ids, layer.ids)


@pytest.mark.parametrize("fmt", [synth.Q3_32, synth.Q3_S256])
def test_fp8_other_formats(fmt):
    base = configs.CONFIGS["decode"]
    cfg = configs.Config("pf8", 1, base.D, base.F, base.E, base.k, 48, fmt, None, None, None)
    wl = configs.build(cfg, device="cuda")
    _check(wl, wl.x, vs_exact=True)


def test_fp8_small_prefill_with_misses():
    # decode-layer shapes with 320/512 resident, 25 tokens (the smallest batches the e4m3 entry takes)
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=25)
    layer, _, _, _ = _check(wl, wl.x)
    assert int(layer.miss_count.item()) > 0


def test_fp8_rejects_small_batches():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=24, layers=1)
    L = wl.layers[0]
    assert moe.workspace_size_fp8(24, wl.cfg.D, wl.cfg.F, wl.cfg.E, wl.cfg.k, wl.cfg.fmt) == 0
    lay = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 24)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_expert_forward_fp8(lay.pool, L.slot_table, wl.x, lay.ids, wl.cfg.k, lay.expert_out, lay.miss_list,
                                   lay.miss_count, moe.alloc_ws(1 << 24))
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def test_fp8_range_bit():
    wl = configs.build(configs.CONFIGS["tiny"], device="cuda", T=32)
    x = wl.x.clone()
    x[3, 7] = 500.0                                        # beyond e4m3's 448
    L = wl.layers[0]
    layer = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 32)
    layer(x, fp8=True)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(layer.ws_fp8) == moe.MOE_ERR_RANGE
