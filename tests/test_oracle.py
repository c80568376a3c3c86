"""Pins of the CPU oracle against facts that do not come from the oracle itself:
hand-worked values, library conversions, exact rational arithmetic, integer
special cases, brute force on tiny inputs and invariants of the method."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests import exact
from tests.packing import Q2_32, Q3_32, Q3_S256, SlotBuilder, build_pool

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FMT = {"q2_32": Q2_32, "q3_32": Q3_32, "q3_s256": Q3_S256}


def bf16_of(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------- number formats
def test_f16_decode_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_to_f32(int(b)) for b in bits[::7]], np.float32)
    r = ref[::7]
    fin = np.isfinite(r)
    assert np.array_equal(got[fin].view(np.uint32), r[fin].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(r))


def test_bf16_rounding_golden():
    with open(os.path.join(GOLDEN, "bf16_rounding.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        assert oracle.bf16_rne(c["value"]) == int(c["bits"], 16), c


def test_bf16_rounding_matches_library_conversion():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(4000).astype(np.float32),
                        (rng.standard_normal(1000) * 1e-39).astype(np.float32),   # subnormals
                        (rng.standard_normal(1000) * 1e30).astype(np.float32)])
    ref = bf16_of(v)
    got = np.array([oracle.bf16_rne(float(x)) for x in v], np.uint16)
    assert np.array_equal(got, ref)
    # doubles that are not float32 values: compare with exact rounding
    for x in rng.standard_normal(300):
        assert oracle.bf16_rne(float(x)) == exact.bf16_bits(exact.bf16(Fraction(float(x))))


# --------------------------------------------------------------- dequantisation
def test_dequant_golden_cases():
    with open(os.path.join(GOLDEN, "dequant_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        fmt = FMT[c["fmt"]]
        D, F = (256, 256) if fmt == Q3_S256 else (32, 32)
        b = SlotBuilder(fmt, D, F)
        n = len(c["codes"])
        b.codes[0][0, :n] = c["codes"]
        if fmt == Q3_S256:
            b.sub[0][0, 0, :] = c["sc"]
            b.d[0][0, 0] = c["d"]
        else:
            b.s[0][0, 0] = c["s"]
            b.m[0][0, 0] = c["m"]
        w = oracle.dequant(build_pool([b]), 0, 0)
        assert w[0, :n].tolist() == c["weights"], c


@pytest.mark.parametrize("fmt", [Q2_32, Q3_32, Q3_S256])
def test_dequant_random_blocks_exact(fmt):
    rng = np.random.default_rng(fmt)
    D, F = (512, 256) if fmt == Q3_S256 else (96, 64)
    b = SlotBuilder(fmt, D, F)
    for i in range(3):
        b.codes[i][:] = rng.integers(0, 1 << (2 if fmt == Q2_32 else 3), b.codes[i].shape)
        if fmt == Q3_S256:
            b.sub[i][:] = rng.integers(0, 64, b.sub[i].shape)
            b.d[i][:] = (rng.random(b.d[i].shape) * 1e-3).astype(np.float16)
        else:
            b.s[i][:] = (rng.random(b.s[i].shape) * 0.05).astype(np.float16)
            b.m[i][:] = (-rng.random(b.m[i].shape) * 0.1).astype(np.float16)
    pool = build_pool([b, b])
    want = b.weights()
    for mat in range(3):
        got = oracle.dequant(pool, 1, mat)
        # s*q + m is exact in double; one rounding to fp32 equals fmaf
        assert np.array_equal(got, want[mat].astype(np.float32)), mat


# --------------------------------------------------------------- router logits
def test_logits_integer_inputs_are_exact():
    rng = np.random.default_rng(1)
    T, D, E = 3, 512, 7
    x = rng.integers(-8, 9, (T, D)).astype(np.float32)
    W = rng.integers(-8, 9, (E, D)).astype(np.float32)
    b = rng.integers(-100, 100, E).astype(np.float32)
    got = oracle.router_logits(bf16_of(x), bf16_of(W), b)
    want = x.astype(np.int64) @ W.astype(np.int64).T + b.astype(np.int64)
    assert np.array_equal(got, want.astype(np.float32))


def test_logits_single_nonzero_element():
    D, E = 256, 4
    x = np.zeros((1, D), np.float32); x[0, 77] = 1.5
    W = np.random.default_rng(2).standard_normal((E, D)).astype(np.float32)
    Wb = bf16_of(W)
    got = oracle.router_logits(bf16_of(x), Wb)
    assert np.array_equal(got[0], (1.5 * bf16_to_f64(Wb[:, 77])).astype(np.float32))


def test_logits_canonical_order_exact_model():
    """Bit-exact against an exact-rational model of the canonical order."""
    rng = np.random.default_rng(3)
    T, D, E = 2, 256, 3
    xb = bf16_of(rng.standard_normal((T, D)))
    Wb = bf16_of(rng.standard_normal((E, D)) * 0.02)
    bias = rng.standard_normal(E).astype(np.float32)
    got = oracle.router_logits(xb, Wb, bias)
    xv = bf16_to_f64(xb); Wv = bf16_to_f64(Wb)
    for t in range(T):
        for e in range(E):
            acc = [Fraction(0)] * 32
            for c in range(D // 256):
                for j in range(8):
                    for L in range(32):
                        i = 256 * c + 8 * L + j
                        acc[L] = exact.fmaf(Fraction(xv[t, i]), Fraction(Wv[e, i]), acc[L])
            half = 16
            while half >= 1:
                for L in range(half):
                    acc[L] = exact.addf(acc[L], acc[L + half])
                half //= 2
            want = exact.addf(acc[0], Fraction(float(bias[e])))
            assert got[t, e] == exact.to_float32(want), (t, e)


def test_logits_error_bound_vs_exact_dot():
    rng = np.random.default_rng(4)
    T, D, E = 4, 3072, 16
    xb = bf16_of(rng.standard_normal((T, D)))
    Wb = bf16_of(rng.standard_normal((E, D)) * 0.02)
    got = oracle.router_logits(xb, Wb).astype(np.float64)
    xv, Wv = bf16_to_f64(xb), bf16_to_f64(Wb)
    exact_dot = xv @ Wv.T                      # products exact in double; error ~1e-16 relative
    mag = np.abs(xv) @ np.abs(Wv).T
    depth = D // 32 + 5
    bound = depth * 2.0 ** -24 * mag * 1.01 + 1e-12
    assert np.all(np.abs(got - exact_dot) <= bound)


# --------------------------------------------------------------- top-k and gates
def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(5)
    T, E, k = 64, 40, 10
    logits = rng.integers(-6, 6, (T, E)).astype(np.float32) * 0.5   # many exact ties
    ids, gates = oracle.topk_gates(logits, k)
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
        assert ids[t].tolist() == order[:k].tolist()
        sel = logits[t, ids[t]]
        rest = np.delete(logits[t], ids[t])
        assert sel.min() >= rest.max()


def test_uniform_logits_closed_form():
    ids, gates = oracle.topk_gates(np.zeros((3, 512), np.float32), 10)
    assert np.array_equal(ids, np.tile(np.arange(10, dtype=np.int32), (3, 1)))
    assert np.all(gates == 1.0 / 10)


def test_gates_k2_closed_form_and_sum():
    rng = np.random.default_rng(6)
    logits = rng.standard_normal((50, 16)).astype(np.float32)
    ids, gates = oracle.topk_gates(logits, 2)
    for t in range(50):
        l0, l1 = float(logits[t, ids[t, 0]]), float(logits[t, ids[t, 1]])
        assert gates[t, 0] == pytest.approx(1.0 / (1.0 + math.exp(l1 - l0)), rel=1e-15)
    ids, gates = oracle.topk_gates(rng.standard_normal((50, 512)).astype(np.float32), 10)
    assert np.allclose(gates.sum(1), 1.0, rtol=0, atol=1e-15)
    assert np.all(np.diff(gates, axis=1) <= 0)


# --------------------------------------------------------------- slot lookup
def test_slot_lookup_brute_force():
    rng = np.random.default_rng(7)
    T, k, E, S = 9, 10, 64, 30
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    table = np.full(E, -1, np.int32)
    table[rng.permutation(E)[:S]] = rng.permutation(S)
    table[3] = 999           # out of range -> miss
    table[5] = -7            # negative -> miss
    slots, miss = oracle.slot_lookup(ids, table, S)
    want_miss = []
    for t in range(T):
        for r in range(k):
            s = table[ids[t, r]]
            ok = 0 <= s < S
            assert slots[t, r] == (s if ok else -1)
            if not ok:
                want_miss.append((t, r, ids[t, r]))
    assert [tuple(m) for m in miss.tolist()] == want_miss


# --------------------------------------------------------------- expert FFN
def _integer_slot(fmt, D, F, rng, big_gate=True):
    """Integer weights: Q2/Q3_32 with s=1, m=0 (w = q); Q3_S256 with d=1, sc=33 (w = q-4)."""
    b = SlotBuilder(fmt, D, F)
    hi = 4 if fmt == Q2_32 else 8
    for i in range(3):
        lo = 1 if (i == 0 and big_gate and fmt != Q3_S256) else 0
        b.codes[i][:] = rng.integers(lo, hi, b.codes[i].shape)
        if fmt == Q3_S256:
            b.sub[i][:] = 33
            b.d[i][:] = 1.0
        else:
            b.s[i][:] = 1.0
            b.m[i][:] = 0.0
    if fmt == Q3_S256 and big_gate:
        b.codes[0][:] = rng.integers(5, 8, b.codes[0].shape)     # w in 1..3
    return b


@pytest.mark.parametrize("fmt", [Q2_32, Q3_32, Q3_S256])
def test_expert_integer_case_reduces_to_matmul(fmt):
    """With gate pre-activations >= 40, silu(g) == g in double, so
    h = bf16(g*u) and y = Wd h are integer matrix products (D != F catches a
    transposed operand, gate/up order is checked by the asymmetry of silu)."""
    rng = np.random.default_rng(10 + fmt)
    D, F = (512, 256) if fmt == Q3_S256 else (96, 64)
    b = _integer_slot(fmt, D, F, rng)
    pool = build_pool([b])
    Wg, Wu, Wd = [w.astype(np.int64) for w in b.weights()]
    x = np.ones(D, np.int64)
    g = Wg @ x
    u = Wu @ x
    assert g.min() >= 40
    h = bf16_of((g * u).astype(np.float32))          # g*u < 2^24: exact fp32, one RNE to bf16
    y = Wd.astype(np.float64) @ bf16_to_f64(h)
    hh, yy = oracle.expert(pool, 0, bf16_of(x.astype(np.float32)))
    assert np.array_equal(hh, h)
    assert np.array_equal(yy, y)


def test_expert_silu_closed_form():
    rng = np.random.default_rng(11)
    D, F = 64, 32
    b = SlotBuilder(Q2_32, D, F)
    for i in range(3):
        b.codes[i][:] = rng.integers(0, 4, b.codes[i].shape)
        b.s[i][:] = 0.03125
        b.m[i][:] = -0.046875
    pool = build_pool([b])
    Wg, Wu, Wd = b.weights()
    x = rng.integers(-3, 4, D).astype(np.float64)
    g, u = Wg @ x, Wu @ x                       # exact: dyadic values with few bits
    hh, yy = oracle.expert(pool, 0, bf16_of(x.astype(np.float32)))
    for f in range(F):
        hv = Fraction(g[f]) / (1 + Fraction(math.exp(-g[f])))
        want = exact.bf16(hv * Fraction(u[f]))
        # silu evaluated in double: allow the neighbouring bf16 value only at a near-tie
        got = exact.bf16_value(hh[f])
        assert abs(got - want) <= abs(want) * Fraction(1, 256) + Fraction(1, 10 ** 30)
    assert np.allclose(yy, Wd @ bf16_to_f64(hh), rtol=1e-14, atol=1e-14)


def test_zero_up_expert_gives_zero():
    rng = np.random.default_rng(12)
    b = _integer_slot(Q2_32, 64, 32, rng)
    b.codes[1][:] = 0                            # Wu = 0 (s=1, m=0)
    h, y = oracle.expert(build_pool([b]), 0, bf16_of(rng.standard_normal(64)))
    assert np.all(bf16_to_f64(h) == 0) and np.all(y == 0)


# --------------------------------------------------------------- whole layer
def _random_pool(rng, n_slots, D=64, F=32, fmt=Q2_32):
    bs = []
    for _ in range(n_slots):
        b = SlotBuilder(fmt, D, F)
        for i in range(3):
            b.codes[i][:] = rng.integers(0, 4, b.codes[i].shape)
            b.s[i][:] = (0.02 * (0.5 + rng.random(b.s[i].shape))).astype(np.float16)
            b.m[i][:] = (-1.5 * b.s[i].astype(np.float32)).astype(np.float16)
        bs.append(b)
    return bs


def _layer_inputs(rng, T, D, E):
    x = bf16_of(rng.standard_normal((T, D)))
    Wr = bf16_of(rng.standard_normal((E, D)) * 0.02)
    return x, Wr


def test_layer_equals_composition_of_experts_with_misses():
    """out = bf16( sum_{hit r} g_r y_r + y_shared ): misses contribute nothing and
    the gates are not renormalised over the hits."""
    rng = np.random.default_rng(13)
    T, D, E, k = 5, 256, 12, 3
    bs = _random_pool(rng, 9, D=D)
    pool = build_pool(bs, shared_slot=8)
    table = np.full(E, -1, np.int32)
    table[:8] = rng.permutation(8)
    x, Wr = _layer_inputs(rng, T, D, E)
    res = oracle.moe_layer(pool, table, k, x, Wr)
    ids, gates = oracle.topk_gates(oracle.router_logits(x, Wr), k)
    assert np.array_equal(res.ids, ids)
    for t in range(T):
        acc = np.zeros(D)
        for r in range(k):
            s = table[ids[t, r]]
            if s >= 0:
                acc += gates[t, r] * oracle.expert(pool, int(s), x[t])[1]
        acc = acc + oracle.expert(pool, 8, x[t])[1]
        want = np.array([exact.bf16_bits(exact.bf16(Fraction(v))) for v in acc], np.uint16)
        assert np.array_equal(res.out[t], want)
    assert len(res.miss_list) == int((table[ids] < 0).sum())


def test_layer_token_permutation_and_slot_relabel_invariance():
    rng = np.random.default_rng(14)
    T, D, E, k = 6, 256, 10, 2
    bs = _random_pool(rng, 11, D=D)
    x, Wr = _layer_inputs(rng, T, D, E)
    table = rng.permutation(10).astype(np.int32)
    base = oracle.moe_layer(build_pool(bs, shared_slot=10), table, k, x, Wr)
    p = rng.permutation(T)
    perm = oracle.moe_layer(build_pool(bs, shared_slot=10), table, k, x[p], Wr)
    assert np.array_equal(perm.out, base.out[p])
    # relabel slots: slot s moves to sigma[s]
    sigma = rng.permutation(11)
    bs2 = [None] * 11
    for s in range(11):
        bs2[sigma[s]] = bs[s]
    relab = oracle.moe_layer(build_pool(bs2, shared_slot=int(sigma[10])), sigma[table].astype(np.int32), k, x, Wr)
    assert np.array_equal(relab.out, base.out)


def test_layer_miss_partial_and_residual_only():
    """With every down projection zero, out = bf16(miss_partial + residual)."""
    rng = np.random.default_rng(15)
    T, D, E, k = 4, 256, 8, 2
    bs = _random_pool(rng, 9, D=D)
    for b in bs:
        b.codes[2][:] = 0
        b.s[2][:] = 0
        b.m[2][:] = 0
    x, Wr = _layer_inputs(rng, T, D, E)
    mp = rng.standard_normal((T, D)).astype(np.float32)
    resid = bf16_of(rng.standard_normal((T, D)))
    table = np.arange(8, dtype=np.int32)
    out = oracle.moe_layer(build_pool(bs, shared_slot=8), table, k, x, Wr, miss_partial=mp, residual=resid).out
    rv = bf16_to_f64(resid)
    for t in range(T):
        want = [exact.bf16_bits(exact.bf16(Fraction(float(mp[t, d])) + Fraction(rv[t, d]))) for d in range(D)]
        assert out[t].tolist() == want


def test_layer_linear_in_down_scale():
    """Doubling one expert's down scale doubles exactly that expert's y."""
    rng = np.random.default_rng(16)
    D = 256
    bs = _random_pool(rng, 2, D=D)
    x = bf16_of(rng.standard_normal(D))
    _, y1 = oracle.expert(build_pool(bs), 1, x)
    bs[1].s[2] = (bs[1].s[2].astype(np.float32) * 2).astype(np.float16)
    bs[1].m[2] = (bs[1].m[2].astype(np.float32) * 2).astype(np.float16)
    _, y2 = oracle.expert(build_pool(bs), 1, x)
    assert np.array_equal(y2, 2 * y1)


def test_dense_reference_all_resident_tiny_config():
    """Tiny config, all 16 experts resident: the layer equals the dense mixture
    sum_e mask(e in topk) g_e y_e + y_shared with every expert evaluated."""
    from bit_expert_ffn_route_b200 import configs
    wl = configs.build(configs.CONFIGS["tiny"])
    pool = oracle.HostPool(wl.pool.fmt, wl.pool.d_model, wl.pool.d_ff, wl.pool.n_slots,
                           wl.layers[0].shared_slot, wl.pool.codes.numpy(), wl.pool.scales.numpy(),
                           wl.pool.stride_codes, wl.pool.stride_scales)
    x = wl.x.view(torch.uint16).numpy()
    Wr = wl.layers[0].Wr.view(torch.uint16).numpy()
    table = wl.layers[0].slot_table.numpy()
    res = oracle.moe_layer(pool, table, 2, x, Wr)
    assert len(res.miss_list) == 0
    # gap >= 1e-2 between the k-th and (k+1)-th logit for every token
    s = -np.sort(-res.logits, axis=1)
    assert (s[:, 1] - s[:, 2]).min() >= 1e-2
    for t in range(x.shape[0]):
        acc = np.zeros(wl.cfg.D)
        for e in range(16):
            r = np.where(res.ids[t] == e)[0]
            if len(r):
                acc += res.gates[t, r[0]] * oracle.expert(pool, int(table[e]), x[t])[1]
        acc += oracle.expert(pool, wl.layers[0].shared_slot, x[t])[1]
        want = np.array([exact.bf16_bits(exact.bf16(Fraction(v))) for v in acc], np.uint16)
        assert np.array_equal(res.out[t], want)
