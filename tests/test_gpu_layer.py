"""GPU parity of the one-call layer (moe_layer_forward, T <= 8): its ids, gates,
miss list, expert rows and output must equal, bit for bit, those of the three
calls moe_route_topk -> moe_expert_forward -> moe_combine (no miss_partial) on
the same inputs; one case is also checked against the CPU oracle directly."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_route_b200 import configs, moe, synth
from tests.harness import oracle_layer, rel_l2_per_token, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    moe.lib()


def _rows_of_hits(layer, T, D, k):
    """The expert-out row map and the rows it points at (fp32), as numpy."""
    raw = layer.expert_out.cpu().numpy()
    rowmap = raw[:T * (k + 1) * 4].view(np.int32).copy()
    off = ((T * (k + 1) * 4 + 255) // 256) * 256
    rows = raw[off:off + T * (k + 1) * D * 4].view(np.float32).reshape(T * (k + 1), D)
    return rowmap, rows[rowmap[rowmap >= 0]].copy()


def _compare(wl, x, k=None, residual=None, layer_idx=0, reps=1):
    k = k or wl.cfg.k
    L = wl.layers[layer_idx]
    T, D = x.shape
    three = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, k, T)
    one = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, k, T)
    out3 = three(x, residual=residual).clone()
    for _ in range(reps):                     # repeated calls on one workspace
        one.out.fill_(0)
        out1 = one.fused(x, residual=residual)
        torch.cuda.synchronize()
        assert moe.moe_workspace_status(one.layer_ws) == moe.MOE_OK
        assert np.array_equal(one.ids.cpu().numpy(), three.ids.cpu().numpy())
        assert np.array_equal(one.gates.cpu().numpy().view(np.uint32), three.gates.cpu().numpy().view(np.uint32))
        n = int(three.miss_count.item())
        assert int(one.miss_count.item()) == n
        assert np.array_equal(one.miss_list[:n].cpu().numpy(), three.miss_list[:n].cpu().numpy())
        map1, rows1 = _rows_of_hits(one, T, D, k)
        map3, rows3 = _rows_of_hits(three, T, D, k)
        assert np.array_equal(map1, map3)
        assert np.array_equal(rows1.view(np.uint32), rows3.view(np.uint32))
        assert np.array_equal(u16(out1), u16(out3))
    return one, three


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8])
def test_layer_matches_three_calls(T):
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=T, layers=1)
    _compare(wl, wl.x)


def test_layer_residual_and_repeats():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", layers=1)
    res = synth.hidden(4, wl.cfg.D, seed=99, device="cuda")
    _compare(wl, wl.x, residual=res, reps=3)


def test_layer_out_aliases_residual():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", layers=1)
    L = wl.layers[0]
    res = synth.hidden(4, wl.cfg.D, seed=5, device="cuda")
    three = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 4)
    ref = three(wl.x, residual=res).clone()
    one = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 4)
    buf = res.clone()
    one.fused(wl.x, residual=buf, out=buf)
    torch.cuda.synchronize()
    assert np.array_equal(u16(buf), u16(ref))


@pytest.mark.parametrize("fmt", [synth.Q3_32, synth.Q3_S256])
@pytest.mark.parametrize("T", [4, 8])
def test_layer_other_formats(fmt, T):
    c = configs.CONFIGS["decode"]
    cfg = configs.Config("layer_f", 1, c.D, c.F, c.E, c.k, T, fmt, [320], 1.1, 0.47)
    wl = configs.build(cfg, device="cuda", layers=1)
    _compare(wl, wl.x)


def test_layer_small_shapes_no_bias():
    # E < #SMs (some CTAs compute no logits), k = 2, no router bias
    wl = configs.build(configs.CONFIGS["tiny"], device="cuda")
    assert wl.layers[0].bias is None
    _compare(wl, wl.x)


def test_layer_every_id_distinct():
    # 8 tokens x top-16 of 128 experts, every expert resident: up to 128 owners
    cfg = configs.Config("layer_owners", 1, 256, 128, 128, 16, 8, synth.Q2_32, None, None, None, seed=3)
    wl = configs.build(cfg, device="cuda")
    _compare(wl, wl.x)


def test_layer_oracle():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", layers=1)
    L = wl.layers[0]
    one = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 4)
    out = one.fused(wl.x)
    torch.cuda.synchronize()
    ref = oracle_layer(wl.pool, L, wl.cfg.k, u16(wl.x))
    assert np.array_equal(one.ids.cpu().numpy(), ref.ids)
    assert rel_l2_per_token(u16(out), ref.out).max() <= 1e-2


def test_layer_dead_workspace_does_no_work():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", layers=1)
    L = wl.layers[0]
    one = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 4)
    one.layer_ws.view(torch.int32)[1] = 1               # the timeout bit, as a give-up leaves it
    one.ids.fill_(-7)
    one.out.fill_(0)
    one.fused(wl.x)
    assert moe.moe_workspace_status(one.layer_ws) == moe.MOE_ERR_TIMEOUT
    assert bool((one.ids == -7).all()) and bool((one.out.view(torch.int16) == 0).all())


def test_layer_rejects_large_batches():
    wl = configs.build(configs.CONFIGS["decode"], device="cuda", T=9, layers=1)
    L = wl.layers[0]
    assert moe.layer_workspace_size(9, wl.cfg.D, wl.cfg.F, wl.cfg.E, wl.cfg.k, wl.cfg.fmt) == 0
    lay = moe.Layer(wl.pool, L.shared_slot, L.slot_table, L.Wr, L.bias, wl.cfg.k, 9)
    ws = moe.alloc_ws(1 << 20)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_layer_forward(lay.pool, L.slot_table, wl.x, L.Wr, L.bias, wl.cfg.k, lay.ids, lay.gates,
                              lay.expert_out, lay.miss_list, lay.miss_count, lay.out, ws)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED
