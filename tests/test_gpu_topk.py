"""GPU top-k selection on shaped logits, decode (T <= 4) and prefill (T > 4)
routers, through the C ABI, against the oracle.

With Wr = 0 every canonical dot product is +0, so the logits equal the bias
exactly; the bias then shapes the selection problem: hot values crowded into a
few lanes of the 32-lane layout (more candidates than one warp holds, the
tournament path), ties broken by the lower id, all-equal logits, E not a
multiple of 32 and E = 1024.  The oracle computes its own logits from the same
inputs (never from the GPU's) and sorts by (logit desc, id asc).  Bars: ids
and logits bit-exact, gates within 1e-6 relative."""
import numpy as np
import pytest
import torch

import oracle
from bit_expert_ffn_route_b200 import moe, synth
from tests.harness import u16

pytestmark = pytest.mark.gpu

TOL_GATE = 1e-6
D = 256


def _bias(kind, E, rng):
    e = np.arange(E)
    if kind == "hot_lanes":      # ids in lanes 0-2 of each 32-block beat all others
        return np.where(e % 32 < 3, 10.0 + e / 1000.0, e / 1.0e6).astype(np.float32)
    if kind == "all_equal":
        return np.zeros(E, np.float32)
    if kind == "ties_stride7":   # a tie class spread over many lanes
        return np.where(e % 7 == 0, 1.0, 0.0).astype(np.float32)
    if kind == "quarter_steps":  # many ties at every level
        return (np.round(rng.random(E) * 4.0) / 4.0).astype(np.float32)
    if kind == "random":
        return rng.standard_normal(E).astype(np.float32)
    raise ValueError(kind)


CASES = [(kind, T, E, k)
         for kind in ("hot_lanes", "all_equal", "ties_stride7", "quarter_steps", "random")
         for T in (4, 8, 12, 64)
         for (E, k) in ((512, 10), (80, 16), (1024, 8))]


@pytest.mark.parametrize("kind,T,E,k", CASES)
def test_topk_on_shaped_logits(kind, T, E, k):
    rng = np.random.default_rng([T, E, k, len(kind)])
    bias = _bias(kind, E, rng)
    x = synth.hidden(T, D, seed=7, stream=E + k, device="cuda")
    Wr = torch.zeros(E, D, dtype=torch.bfloat16, device="cuda")
    b = torch.from_numpy(bias).cuda()
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gates = torch.empty(T, k, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ws = moe.alloc_ws(moe.route_workspace_size(T, D, E, k))
    moe.moe_route_topk(x, Wr, b, k, ids, gates, ws, logits=logits)
    torch.cuda.synchronize()
    ref_logits = oracle.router_logits(u16(x), u16(Wr), bias)
    ref_ids, ref_gates = oracle.topk_gates(ref_logits, k)
    assert np.array_equal(logits.cpu().numpy().view(np.uint32), ref_logits.view(np.uint32))
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    g = gates.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - ref_gates) <= TOL_GATE * np.abs(ref_gates))
    assert int(ws[4:8].view(torch.int32).item()) == 0
