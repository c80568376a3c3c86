"""moe_route_topk_static: the router entry point for callers that cannot
allocate device memory themselves (for example code whose host framework owns
all GPU memory through a fixed arena, or code that must not call cudaMalloc
while a stream is being captured).  It keeps its scratch in a library-owned
static device array instead of a caller-provided workspace.

The tests call it through the C ABI twice in a row (and captured in a CUDA
graph, replayed) and check each result
against the workspace-taking moe_route_topk on the same inputs: expert ids and
logits identical, gates within the 1e-6 relative tolerance the other GPU tests
use.  It also checks ragged shapes against the CPU oracle directly, and that
sizes beyond the static array are refused."""
import numpy as np
import pytest
import torch

import oracle
from bit_expert_ffn_route_b200 import configs, moe, synth
from tests.harness import u16

pytestmark = pytest.mark.gpu

TOL_GATE = 1e-6


def test_static_router_matches_workspace_router_twice():
    cfg = configs.CONFIGS["decode"]
    wl = configs.build(cfg, device="cuda", layers=1)
    L = wl.layers[0]
    T, E, D, k = cfg.T, cfg.E, cfg.D, cfg.k
    ws = moe.alloc_ws(moe.route_workspace_size(T, D, E, k))
    for call in range(2):
        x = synth.hidden(T, D, seed=cfg.seed, stream=500 + call, device="cuda")
        ids_a = torch.empty(T, k, dtype=torch.int32, device="cuda")
        gates_a = torch.empty(T, k, dtype=torch.float32, device="cuda")
        logits_a = torch.empty(T, E, dtype=torch.float32, device="cuda")
        ids_b, gates_b, logits_b = torch.empty_like(ids_a), torch.empty_like(gates_a), torch.empty_like(logits_a)
        moe.moe_route_topk(x, L.Wr, L.bias, k, ids_a, gates_a, ws, logits=logits_a)
        moe.moe_route_topk_static(x, L.Wr, L.bias, k, ids_b, gates_b, logits=logits_b)
        ids_c, gates_c = torch.empty_like(ids_a), torch.empty_like(gates_a)
        moe.moe_route_topk_static(x, L.Wr, L.bias, k, ids_c, gates_c)          # logits kept in the static scratch
        torch.cuda.synchronize()
        assert torch.equal(ids_a, ids_b) and torch.equal(ids_a, ids_c), call
        assert torch.equal(logits_a.view(torch.int32), logits_b.view(torch.int32)), call
        ga = gates_a.double().cpu().numpy()
        for g in (gates_b, gates_c):
            assert np.all(np.abs(g.double().cpu().numpy() - ga) <= TOL_GATE * np.abs(ga)), call


def test_static_router_refuses_sizes_beyond_its_array():
    Wr = torch.zeros(512, 3072, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(5, 3072, dtype=torch.bfloat16, device="cuda")         # T = 5 > 4
    ids = torch.empty(5, 10, dtype=torch.int32, device="cuda")
    gates = torch.empty(5, 10, dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route_topk_static(x, Wr, None, 10, ids, gates)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED
    Wr2 = torch.zeros(1100, 3072, dtype=torch.bfloat16, device="cuda")   # E = 1100 > 1024
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route_topk_static(x[:4], Wr2, None, 10, ids[:4], gates[:4])
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("T,E,k", [(1, 18, 4), (3, 18, 4), (2, 1024, 16)])
def test_static_router_ragged_shapes_match_oracle(T, E, k):
    D = 256
    x = synth.hidden(T, D, seed=11, stream=T, device="cuda")
    Wr = synth.router_weight(E, D, seed=11, layer=E, device="cuda")
    bias = synth.zipf_bias(E, 1.1, 0.5, seed=11).cuda()
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gates = torch.empty(T, k, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    for call in range(2):
        moe.moe_route_topk_static(x, Wr, bias, k, ids, gates, logits=logits)
        torch.cuda.synchronize()
        want_l = oracle.router_logits(u16(x), u16(Wr), bias.cpu().numpy())
        want_ids, want_g = oracle.topk_gates(want_l, k)
        assert np.array_equal(logits.cpu().numpy().view(np.uint32), want_l.view(np.uint32)), call
        assert np.array_equal(ids.cpu().numpy(), want_ids), call
        g = gates.double().cpu().numpy()
        assert np.all(np.abs(g - want_g) <= TOL_GATE * np.abs(want_g)), call


def test_static_router_under_graph_capture():
    """The use its header names: one call before any capture, then calls
    captured in a CUDA graph (each issues its memset on the stream) and the
    graph replayed; ids and logits identical to the workspace router."""
    cfg = configs.CONFIGS["decode"]
    wl = configs.build(cfg, device="cuda", layers=1)
    L = wl.layers[0]
    T, E, D, k = cfg.T, cfg.E, cfg.D, cfg.k
    xs = [synth.hidden(T, D, seed=cfg.seed, stream=700 + i, device="cuda") for i in range(2)]
    ids = [torch.empty(T, k, dtype=torch.int32, device="cuda") for _ in range(2)]
    gates = [torch.empty(T, k, dtype=torch.float32, device="cuda") for _ in range(2)]
    logits = [torch.empty(T, E, dtype=torch.float32, device="cuda") for _ in range(2)]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        moe.moe_route_topk_static(xs[0], L.Wr, L.bias, k, ids[0], gates[0], stream=stream)   # before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(2):
            moe.moe_route_topk_static(xs[i], L.Wr, L.bias, k, ids[i], gates[i], logits=logits[i], stream=stream)
    ws = moe.alloc_ws(moe.route_workspace_size(T, D, E, k))
    for rep in range(2):
        for i in range(2):
            ids[i].fill_(-5)
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        for i in range(2):
            ids_a = torch.empty(T, k, dtype=torch.int32, device="cuda")
            gates_a = torch.empty(T, k, dtype=torch.float32, device="cuda")
            logits_a = torch.empty(T, E, dtype=torch.float32, device="cuda")
            moe.moe_route_topk(xs[i], L.Wr, L.bias, k, ids_a, gates_a, ws, logits=logits_a)
            torch.cuda.synchronize()
            assert torch.equal(ids[i], ids_a), (rep, i)
            assert torch.equal(logits[i].view(torch.int32), logits_a.view(torch.int32)), (rep, i)
            ga = gates_a.double().cpu().numpy()
            assert np.all(np.abs(gates[i].double().cpu().numpy() - ga) <= TOL_GATE * np.abs(ga)), (rep, i)
    del g
