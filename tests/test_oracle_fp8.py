"""Pins of the oracle's e4m3-operand variant (orc_e4m3_rne, orc_f16_round,
orc_expert_fp8) against things that share nothing with it: the e4m3 value table
built here from the format's fields with exact fractions (brute-force nearest
value, ties to the even code), torch's float8_e4m3fn cast, numpy's float16
cast, and integer experts in which every operand rounding is exact."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests.packing import Q2_32, Q3_S256, SlotBuilder, build_pool

# e4m3: sign, 4 exponent bits (bias 7), 3 mantissa bits; S.1111.111 is NaN
_FINITE = {}
for _b in range(256):
    _e, _m = (_b >> 3) & 15, _b & 7
    if _e == 15 and _m == 7:
        continue
    _v = Fraction(_m, 512) if _e == 0 else Fraction(8 + _m, 8) * Fraction(2) ** (_e - 7)
    _FINITE[_b] = -_v if _b & 0x80 else _v


def nearest_e4m3(v: Fraction) -> int:
    """The finite e4m3 code nearest to v; ties to the even mantissa; +-0 by sign."""
    cands = [b for b in _FINITE if (b & 0x80) == (0x80 if v < 0 else 0)]
    best = min(abs(_FINITE[b] - v) for b in cands)
    near = [b for b in cands if abs(_FINITE[b] - v) == best]
    if len(near) > 1:
        near = [b for b in near if (b & 1) == 0]
    return near[0]


def test_e4m3_table_round_trip():
    assert len(_FINITE) == 254 and max(_FINITE.values()) == 448 and min(v for v in _FINITE.values() if v > 0) == Fraction(1, 512)
    for b, v in _FINITE.items():
        assert oracle.e4m3_to_f64(b) == float(v)
        if b != 0x80:                                  # -0: a fraction has no sign
            assert oracle.e4m3_rne(float(v)) == b, hex(b)
    assert oracle.e4m3_rne(-0.0) == 0x80
    assert np.isnan(oracle.e4m3_to_f64(0x7F)) and np.isnan(oracle.e4m3_to_f64(0xFF))


def test_e4m3_rounding_brute_force_and_ties():
    rng = np.random.default_rng(7)
    mags = np.exp2(rng.uniform(-12, 9.2, 4000))
    vals = list(mags * rng.choice([-1.0, 1.0], mags.size))
    srt = sorted(set(_FINITE.values()))
    vals += [float((a + b) / 2) for a, b in zip(srt[:-1], srt[1:])]       # every tie
    vals += [460.0, 464.0, 500.0, 1e6, -1e6, 2.0 ** -10, -(2.0 ** -10)]    # saturation, tie to zero
    for v in vals:
        assert oracle.e4m3_rne(v) == nearest_e4m3(Fraction(v)), v


def test_e4m3_matches_torch_cast():
    rng = np.random.default_rng(8)
    v = (np.exp2(rng.uniform(-11, 8.85, 20000)) * rng.choice([-1.0, 1.0], 20000)).astype(np.float32)
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne(float(a)) for a in v], np.uint8)
    assert np.array_equal(got, want)


def test_f16_round_matches_numpy_cast():
    rng = np.random.default_rng(9)
    v = np.exp2(rng.uniform(-26, 15.9, 20000)) * rng.choice([-1.0, 1.0], 20000)
    want = v.astype(np.float16).astype(np.float64)
    got = np.array([oracle.f16_round(float(a)) for a in v])
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", [Q2_32, Q3_S256])
def test_expert_fp8_integer_case_is_exact(fmt):
    """Integer weights (64 w is an e4m3 value: 0..192 or -256..192) and integer
    x in 1..2 (e4m3 values): the gate and up products are exact, gate >= 40 so
    silu(g) == g in double, and h8 = nearest e4m3 of the integer g*u (including
    saturation at 448) is computed here exactly; y = Wd h8 exactly."""
    rng = np.random.default_rng(20 + fmt)
    D, F = (512, 256) if fmt == Q3_S256 else (64, 32)
    b = SlotBuilder(fmt, D, F)
    for i in range(3):
        if fmt == Q3_S256:
            b.sub[i][:] = 33
            b.d[i][:] = 1.0
        else:
            b.s[i][:] = 1.0
            b.m[i][:] = 0.0
    if fmt == Q3_S256:
        b.codes[0][:] = rng.integers(5, 8, b.codes[0].shape)                 # gate w in 1..3
        b.codes[1][:] = np.where(rng.random(b.codes[1].shape) < 0.02, 5, 4)  # up w mostly 0, a few 1
        b.codes[2][:] = rng.integers(0, 8, b.codes[2].shape)                 # down w in -4..3
    else:
        b.codes[0][:] = rng.integers(1, 4, b.codes[0].shape)
        b.codes[1][:] = np.where(rng.random(b.codes[1].shape) < 0.05, 1, 0)
        b.codes[2][:] = rng.integers(0, 4, b.codes[2].shape)
    pool = build_pool([b])
    Wg, Wu, Wd = [w.astype(np.int64) for w in b.weights()]
    x = rng.integers(1, 3, D).astype(np.int64)
    g, u = Wg @ x, Wu @ x
    assert g.min() >= 40 and np.abs(g * u).max() > 448                  # saturation is exercised
    h8 = np.array([float(_FINITE[nearest_e4m3(Fraction(int(gi * ui)))]) for gi, ui in zip(g, u)])
    want = Wd.astype(np.float64) @ h8
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()
    got = oracle.expert_fp8(pool, 0, xb)
    assert np.array_equal(got, want)


def test_expert_fp8_random_vs_library_roundings():
    """Random Q2 expert: the operand roundings done by numpy's float16 cast and
    torch's e4m3 cast, the contractions by numpy matmul in double."""
    rng = np.random.default_rng(31)
    D, F = 256, 64
    b = SlotBuilder(Q2_32, D, F)
    for i in range(3):
        b.codes[i][:] = rng.integers(0, 4, b.codes[i].shape)
        s = (0.02 * (0.5 + rng.random(b.s[i].shape))).astype(np.float16)
        b.s[i][:] = s
        b.m[i][:] = (-1.5 * s.astype(np.float32)).astype(np.float16)
    pool = build_pool([b])

    def e4(a):
        return torch.from_numpy(np.asarray(a, np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()

    W8 = [e4((64.0 * oracle.dequant(pool, 0, m).astype(np.float64)).astype(np.float16).astype(np.float32))
          for m in range(3)]
    x = rng.standard_normal(D).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    x8 = e4(xb.to(torch.float32).numpy())
    g, u = W8[0] @ x8 / 64.0, W8[1] @ x8 / 64.0
    h8 = e4((g / (1.0 + np.exp(-g)) * u).astype(np.float32))
    want = W8[2] @ h8 / 64.0
    got = oracle.expert_fp8(pool, 0, xb.view(torch.uint16).numpy())
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)
