"""The C-ABI library loads and exports every symbol include/*.h declares;
size queries and argument checks behave as documented (no GPU needed: these
calls return before touching the device)."""
import ctypes
import os
import re

import pytest

import oracle
from bit_expert_ffn_route_b200 import build, moe, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return moe.lib()


def declared_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", txt))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(moe.EXPORTS)


@pytest.mark.parametrize("fmt", [synth.Q2_32, synth.Q3_32, synth.Q3_S256])
def test_slot_sizes_agree(L, fmt):
    for D, F in [(3072, 512), (256, 256)]:
        assert L.moe_slot_code_bytes(fmt, D, F) == synth.slot_code_bytes(fmt, D, F) == oracle.slot_code_bytes(fmt, D, F)
        assert L.moe_slot_scale_bytes(fmt, D, F) == synth.slot_scale_bytes(fmt, D, F) == oracle.slot_scale_bytes(fmt, D, F)
    assert L.moe_slot_code_bytes(7, 3072, 512) == 0


def test_size_queries(L):
    assert L.moe_expert_out_size(4, 3072, 10) >= 4 * 11 * 3072 * 4
    assert L.moe_route_workspace_size(4, 3072, 512, 10) >= 256
    assert L.moe_workspace_size(4, 3072, 512, 512, 10, 0) > 0
    assert L.moe_workspace_size(4, 3000, 512, 512, 10, 0) == 0      # D % 256 != 0
    assert L.moe_route_workspace_size(4, 3072, 512, 17) == 0        # k > 16


def test_status_strings(L):
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert L.moe_status_string(s)


def _fake(addr=1 << 20):
    return ctypes.c_void_p(addr)


def test_route_argument_errors(L):
    f = _fake()
    # shape errors first
    assert L.moe_route_topk(f, 4, 3000, f, None, 512, 10, f, f, None, f, 1 << 20, None) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_route_topk(f, 4, 3072, f, None, 512, 0, f, f, None, f, 1 << 20, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(f, 4, 3072, f, None, 8, 10, f, f, None, f, 1 << 20, None) == moe.MOE_ERR_UNSUPPORTED
    # null / misaligned pointers
    assert L.moe_route_topk(None, 4, 3072, f, None, 512, 10, f, f, None, f, 1 << 20, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(_fake((1 << 20) + 2), 4, 3072, f, None, 512, 10, f, f, None, f, 1 << 20, None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    assert L.moe_route_topk(f, 4, 3072, f, None, 512, 10, f, f, None, f, 16, None) == moe.MOE_ERR_WORKSPACE
    # T == 0 is a no-op
    assert L.moe_route_topk(None, 0, 3072, None, None, 512, 10, None, None, None, None, 0, None) == moe.MOE_OK


def _pool(fmt=0, D=3072, F=512, n=4, shared=0, stride_c=None, stride_s=None):
    f = fmt if fmt in (0, 1, 2) else 0
    sc = stride_c if stride_c is not None else -(-synth.slot_code_bytes(f, D, F) // 256) * 256
    ss = stride_s if stride_s is not None else -(-synth.slot_scale_bytes(f, D, F) // 256) * 256
    return moe.moe_pool(fmt, D, F, n, shared, 0, 1 << 30, 1 << 31, sc, ss)


def test_forward_argument_errors(L):
    f = _fake()
    fw = lambda pool, T=4, E=512, k=10, eo=1 << 30, ws=1 << 30: L.moe_expert_forward(
        ctypes.byref(pool), f, E, f, T, f, k, f, eo, f, f, f, ws, None)
    assert fw(_pool(fmt=5)) == moe.MOE_ERR_INVALID_ARG
    assert fw(_pool(shared=4)) == moe.MOE_ERR_INVALID_ARG
    assert fw(_pool(D=3000)) == moe.MOE_ERR_UNSUPPORTED
    assert fw(_pool(F=200)) == moe.MOE_ERR_UNSUPPORTED
    assert fw(_pool(fmt=2, F=384)) == moe.MOE_ERR_UNSUPPORTED
    assert fw(_pool(stride_c=256)) == moe.MOE_ERR_INVALID_ARG          # stride below slot size
    assert fw(_pool(stride_c=1769472 + 8)) == moe.MOE_ERR_INVALID_ARG  # not a multiple of 256
    assert fw(_pool(), k=17) == moe.MOE_ERR_UNSUPPORTED
    assert fw(_pool(), eo=16) == moe.MOE_ERR_WORKSPACE
    assert fw(_pool(), ws=16) == moe.MOE_ERR_WORKSPACE
    bad = _pool()
    bad.reserved = 1
    assert fw(bad) == moe.MOE_ERR_INVALID_ARG
    # null miss_count
    assert L.moe_expert_forward(ctypes.byref(_pool()), f, 512, f, 4, f, 10, f, 1 << 30, f, None, f, 1 << 30,
                                None) == moe.MOE_ERR_INVALID_ARG


def test_combine_and_dequant_argument_errors(L):
    f = _fake()
    assert L.moe_combine(f, f, 4, 3000, 10, None, None, f, None) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_combine(None, f, 4, 3072, 10, None, None, f, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(f, f, -1, 3072, 10, None, None, f, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(None, None, 0, 3072, 10, None, None, None, None) == moe.MOE_OK
    assert L.moe_dequantize(ctypes.byref(_pool()), 4, 0, f, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dequantize(ctypes.byref(_pool()), 0, 3, f, None) == moe.MOE_ERR_INVALID_ARG


def test_cache_call_argument_errors(L):
    f = _fake()
    # popularity count: shape / pointer errors, and T == 0 launches nothing
    assert L.moe_expert_hist(f, 4, 0, 512, f, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_hist(f, 4, 10, 0, f, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_hist(None, 4, 10, 512, f, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_hist(f, 4, 10, 512, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_hist(None, 0, 10, 512, None, None) == moe.MOE_OK
    # slot fill: bad pool, slot or host pointers are refused before any copy
    fill = lambda pool, slot=0, hc=f, hs=f: L.moe_slot_fill(ctypes.byref(pool), slot, hc, hs, None)
    assert fill(_pool(fmt=5)) == moe.MOE_ERR_INVALID_ARG
    assert fill(_pool(), slot=4) == moe.MOE_ERR_INVALID_ARG
    assert fill(_pool(), slot=-1) == moe.MOE_ERR_INVALID_ARG
    assert fill(_pool(), hc=None) == moe.MOE_ERR_INVALID_ARG
    assert fill(_pool(stride_c=256)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_slot_fill(None, 0, f, f, None) == moe.MOE_ERR_INVALID_ARG


def test_status_query_and_wait_hook_argument_errors(L):
    f = _fake()
    assert L.moe_workspace_status(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_status(_fake((1 << 20) + 16), None) == moe.MOE_ERR_INVALID_ARG   # not 256-aligned
    assert L.moe_debug_wait_flag(None, 1, 1000, f, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_debug_wait_flag(f, 1, 1000, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_debug_wait_flag(f, 1, 0, f, None) == moe.MOE_ERR_INVALID_ARG             # no limit
    assert L.moe_debug_wait_flag(f, 1, 2000000, f, None) == moe.MOE_ERR_INVALID_ARG       # above 1 s


def test_operand_hook_argument_errors(L):
    f = _fake()
    assert L.moe_debug_operand_workspace_size(3072, 512) > 128 * 3072 * 2
    op = lambda pool=_pool(), gemm=1, slot=0, m0=0, dump=f, ws=f, nb=1 << 30: L.moe_debug_prefill_operand(
        ctypes.byref(pool), gemm, slot, m0, dump, ws, nb, None)
    assert op(gemm=3) == moe.MOE_ERR_INVALID_ARG
    assert op(slot=4) == moe.MOE_ERR_INVALID_ARG
    assert op(m0=32) == moe.MOE_ERR_INVALID_ARG            # gate|up tiles start at multiples of 128
    assert op(m0=64) == moe.MOE_ERR_INVALID_ARG
    assert op(gemm=2, m0=64) == moe.MOE_ERR_INVALID_ARG    # down tiles start at multiples of 256
    assert op(gemm=2, m0=128) == moe.MOE_ERR_INVALID_ARG
    assert op(m0=512) == moe.MOE_ERR_INVALID_ARG           # beyond d_ff
    assert op(dump=None) == moe.MOE_ERR_INVALID_ARG
    assert op(nb=64) == moe.MOE_ERR_WORKSPACE


def test_layer_size_and_argument_errors(L):
    assert L.moe_layer_workspace_size(4, 3072, 512, 512, 10, 0) >= 1024 + 32768
    assert L.moe_layer_workspace_size(8, 3072, 512, 512, 10, 2) > L.moe_layer_workspace_size(4, 3072, 512, 512, 10, 2)
    assert L.moe_layer_workspace_size(9, 3072, 512, 512, 10, 0) == 0      # one call covers T <= 8
    assert L.moe_layer_workspace_size(4, 3000, 512, 512, 10, 0) == 0
    f, g = _fake(), _fake(1 << 21)
    lf = lambda pool, T=4, E=512, k=10, eo=1 << 30, ws=1 << 30, x=f, out=g: L.moe_layer_forward(
        ctypes.byref(pool), f, E, x, T, f, None, k, f, f, f, eo, f, f, None, out, f, ws, None)
    assert lf(_pool(fmt=5)) == moe.MOE_ERR_INVALID_ARG
    assert lf(_pool(D=3000)) == moe.MOE_ERR_UNSUPPORTED
    assert lf(_pool(), T=9) == moe.MOE_ERR_UNSUPPORTED
    assert lf(_pool(), k=17) == moe.MOE_ERR_UNSUPPORTED
    assert lf(_pool(), eo=16) == moe.MOE_ERR_WORKSPACE
    assert lf(_pool(), ws=16) == moe.MOE_ERR_WORKSPACE
    assert lf(_pool(), out=None) == moe.MOE_ERR_INVALID_ARG
    assert lf(_pool(), x=f, out=f) == moe.MOE_ERR_INVALID_ARG        # out may not alias x


def test_small_batch_layout_and_fp8_entry(L):
    """Batches of up to 24 tokens take the decode path (fp32 rows in expert_out,
    a workspace for 8-token launches); the e4m3 entry takes only larger ones."""
    D, F, E, k = 3072, 512, 512, 10
    rowmap = lambda T: (T * (k + 1) * 4 + 255) // 256 * 256
    assert L.moe_expert_out_size(24, D, k) == rowmap(24) + 24 * (k + 1) * D * 4
    assert L.moe_expert_out_size(25, D, k) == rowmap(25) + 25 * (k + 1) * D * 2
    assert L.moe_workspace_size(24, D, F, E, k, 0) == L.moe_workspace_size(8, D, F, E, k, 0)
    assert L.moe_workspace_size(16, D, F, E, k, 0) == L.moe_workspace_size(8, D, F, E, k, 0)
    assert L.moe_workspace_size(25, D, F, E, k, 0) > L.moe_workspace_size(24, D, F, E, k, 0)
    assert L.moe_workspace_size_fp8(24, D, F, E, k, 0) == 0
    assert L.moe_workspace_size_fp8(25, D, F, E, k, 0) == L.moe_workspace_size(25, D, F, E, k, 0)
    f = _fake()
    fw = lambda pool, T=32, eo=1 << 30, ws=1 << 30: L.moe_expert_forward_fp8(
        ctypes.byref(pool), f, E, f, T, f, k, f, eo, f, f, f, ws, None)
    assert fw(_pool(fmt=5)) == moe.MOE_ERR_INVALID_ARG
    assert fw(_pool(), T=24) == moe.MOE_ERR_UNSUPPORTED
    assert fw(_pool(), T=1) == moe.MOE_ERR_UNSUPPORTED
    assert fw(_pool(), eo=16) == moe.MOE_ERR_WORKSPACE
    assert fw(_pool(), ws=16) == moe.MOE_ERR_WORKSPACE
