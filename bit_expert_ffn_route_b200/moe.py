"""Thin ctypes binding of ``libmoe.so`` (include/moe.h).

Argument marshalling only: every step of the expert pass runs in the CUDA
library.  Tensors are torch CUDA tensors; their device pointers and the current
stream are passed straight through.  Loading fails loudly when the library is
missing — there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

from . import synth

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_RANGE = \
    0, -1, -2, -3, -4, -5, -6
MOE_Q2_32, MOE_Q3_32, MOE_Q3_S256 = 0, 1, 2

EXPORTS = ["moe_slot_code_bytes", "moe_slot_scale_bytes", "moe_route_workspace_size", "moe_workspace_size",
           "moe_expert_out_size", "moe_route_topk", "moe_expert_forward", "moe_combine", "moe_dequantize",
           "moe_status_string", "moe_route_topk_static", "moe_expert_hist", "moe_cache_plan", "moe_slot_fill",
           "moe_workspace_status", "moe_debug_wait_flag", "moe_debug_operand_workspace_size",
           "moe_debug_prefill_operand", "moe_layer_workspace_size", "moe_layer_forward",
           "moe_workspace_size_fp8", "moe_expert_forward_fp8"]


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({_lib_status_string(status)})")


class moe_pool(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("n_slots", ctypes.c_int32), ("shared_slot", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("slot_stride_codes", ctypes.c_uint64), ("slot_stride_scales", ctypes.c_uint64)]


_lib = None


def lib():
    """Load libmoe.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m bit_expert_ffn_route_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        for name in ("moe_slot_code_bytes", "moe_slot_scale_bytes"):
            getattr(L, name).restype = sz
            getattr(L, name).argtypes = [i, i, i]
        L.moe_route_workspace_size.restype = sz
        L.moe_route_workspace_size.argtypes = [i, i, i, i]
        L.moe_workspace_size.restype = sz
        L.moe_workspace_size.argtypes = [i, i, i, i, i, i]
        L.moe_expert_out_size.restype = sz
        L.moe_expert_out_size.argtypes = [i, i, i]
        L.moe_route_topk.restype = i
        L.moe_route_topk.argtypes = [P, i, i, P, P, i, i, P, P, P, P, sz, P]
        L.moe_expert_forward.restype = i
        L.moe_expert_forward.argtypes = [ctypes.POINTER(moe_pool), P, i, P, i, P, i, P, sz, P, P, P, sz, P]
        L.moe_expert_forward_fp8.restype = i
        L.moe_expert_forward_fp8.argtypes = [ctypes.POINTER(moe_pool), P, i, P, i, P, i, P, sz, P, P, P, sz, P]
        L.moe_workspace_size_fp8.restype = sz
        L.moe_workspace_size_fp8.argtypes = [i, i, i, i, i, i]
        L.moe_combine.restype = i
        L.moe_combine.argtypes = [P, P, i, i, i, P, P, P, P]
        L.moe_dequantize.restype = i
        L.moe_dequantize.argtypes = [ctypes.POINTER(moe_pool), i, i, P, P]
        L.moe_route_topk_static.restype = i
        L.moe_route_topk_static.argtypes = [P, i, i, P, P, i, i, P, P, P, P]
        L.moe_expert_hist.restype = i
        L.moe_expert_hist.argtypes = [P, i, i, i, P, P]
        L.moe_cache_plan.restype = i
        L.moe_cache_plan.argtypes = [P, i, P, P, i, ctypes.c_float, i, P, P]
        L.moe_slot_fill.restype = i
        L.moe_slot_fill.argtypes = [ctypes.POINTER(moe_pool), i, P, P, P]
        L.moe_workspace_status.restype = i
        L.moe_workspace_status.argtypes = [P, P]
        L.moe_debug_wait_flag.restype = i
        L.moe_debug_wait_flag.argtypes = [P, ctypes.c_uint32, ctypes.c_uint32, P, P]
        L.moe_debug_operand_workspace_size.restype = sz
        L.moe_debug_operand_workspace_size.argtypes = [i, i]
        L.moe_debug_prefill_operand.restype = i
        L.moe_debug_prefill_operand.argtypes = [ctypes.POINTER(moe_pool), i, i, i, P, P, sz, P]
        L.moe_layer_workspace_size.restype = sz
        L.moe_layer_workspace_size.argtypes = [i, i, i, i, i, i]
        L.moe_layer_forward.restype = i
        L.moe_layer_forward.argtypes = [ctypes.POINTER(moe_pool), P, i, P, i, P, P, i, P, P, P, sz, P, P, P, P, P, sz,
                                        P]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [i]
        _lib = L
    return _lib


def _lib_status_string(s):
    try:
        return lib().moe_status_string(int(s)).decode()
    except Exception:
        return "?"


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, st):
    if st != MOE_OK:
        raise MoeError(fn, st)


def make_pool(pool: synth.PoolData, shared_slot: int) -> moe_pool:
    return moe_pool(pool.fmt, pool.d_model, pool.d_ff, pool.n_slots, int(shared_slot), 0,
                    pool.codes.data_ptr(), pool.scales.data_ptr(), pool.stride_codes, pool.stride_scales)


def route_workspace_size(T, D, E, k) -> int:
    return int(lib().moe_route_workspace_size(T, D, E, k))


def workspace_size(T, D, F, E, k, fmt) -> int:
    return int(lib().moe_workspace_size(T, D, F, E, k, fmt))


def layer_workspace_size(T, D, F, E, k, fmt) -> int:
    return int(lib().moe_layer_workspace_size(T, D, F, E, k, fmt))


def expert_out_size(T, D, k) -> int:
    return int(lib().moe_expert_out_size(T, D, k))


def alloc_ws(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled, 256-byte aligned device scratch buffer."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def moe_route_topk(x, Wr, bias, k, ids, gates, ws, logits=None, stream=None):
    T, D = x.shape
    E = Wr.shape[0]
    st = lib().moe_route_topk(_p(x), T, D, _p(Wr), _p(bias), E, k, _p(ids), _p(gates), _p(logits),
                              _p(ws), ws.numel(), _stream(stream))
    _check("moe_route_topk", st)


def moe_route_topk_static(x, Wr, bias, k, ids, gates, logits=None, stream=None):
    """moe_route_topk with library-owned static scratch (T <= 4, E <= 1024)."""
    T, D = x.shape
    E = Wr.shape[0]
    st = lib().moe_route_topk_static(_p(x), T, D, _p(Wr), _p(bias), E, k, _p(ids), _p(gates), _p(logits),
                                     _stream(stream))
    _check("moe_route_topk_static", st)


def moe_expert_forward(pool: moe_pool, slot_table, x, ids, k, expert_out, miss_list, miss_count, ws, stream=None):
    T = x.shape[0]
    E = slot_table.shape[0]
    st = lib().moe_expert_forward(ctypes.byref(pool), _p(slot_table), E, _p(x), T, _p(ids), k,
                                  _p(expert_out), expert_out.numel(), _p(miss_list), _p(miss_count),
                                  _p(ws), ws.numel(), _stream(stream))
    _check("moe_expert_forward", st)


def moe_expert_forward_fp8(pool: moe_pool, slot_table, x, ids, k, expert_out, miss_list, miss_count, ws,
                           stream=None):
    """The expert pass with e4m3 tensor-core operands (lossy; T > 24: smaller batches take the decode path)."""
    T = x.shape[0]
    E = slot_table.shape[0]
    st = lib().moe_expert_forward_fp8(ctypes.byref(pool), _p(slot_table), E, _p(x), T, _p(ids), k,
                                      _p(expert_out), expert_out.numel(), _p(miss_list), _p(miss_count),
                                      _p(ws), ws.numel(), _stream(stream))
    _check("moe_expert_forward_fp8", st)


def workspace_size_fp8(T, D, F, E, k, fmt):
    return lib().moe_workspace_size_fp8(T, D, F, E, k, fmt)


def moe_layer_forward(pool: moe_pool, slot_table, x, Wr, bias, k, ids, gates, expert_out, miss_list, miss_count,
                      out, ws, residual=None, stream=None):
    """The one-call layer (T <= 8): routing, expert pass and combine in one launch."""
    T = x.shape[0]
    E = slot_table.shape[0]
    st = lib().moe_layer_forward(ctypes.byref(pool), _p(slot_table), E, _p(x), T, _p(Wr), _p(bias), k, _p(ids),
                                 _p(gates), _p(expert_out), expert_out.numel(), _p(miss_list), _p(miss_count),
                                 _p(residual), _p(out), _p(ws), ws.numel(), _stream(stream))
    _check("moe_layer_forward", st)


def moe_combine(expert_out, gates, T, D, k, out, miss_partial=None, residual=None, stream=None):
    st = lib().moe_combine(_p(expert_out), _p(gates), T, D, k, _p(miss_partial), _p(residual), _p(out),
                           _stream(stream))
    _check("moe_combine", st)


def moe_workspace_status(ws, stream=None) -> int:
    """The device error word of a workspace as a status code (synchronises the stream)."""
    return int(lib().moe_workspace_status(_p(ws), _stream(stream)))


def moe_debug_wait_flag(flag, expect, limit_us, ws, stream=None):
    """Test hook: a bounded device wait for flag[0] == expect (flag: int32/uint32 device tensor)."""
    _check("moe_debug_wait_flag", lib().moe_debug_wait_flag(_p(flag), int(expect), int(limit_us), _p(ws),
                                                            _stream(stream)))


def moe_debug_prefill_operand(pool: moe_pool, gemm, slot, m0, dump, stream=None):
    """Test hook: the dequantised A operand of one prefill GEMM tile as read back
    from tensor memory.  dump: uint32 device tensor of K/128 * 128 * 64 words."""
    nb = int(lib().moe_debug_operand_workspace_size(pool.d_model, pool.d_ff))
    ws = alloc_ws(nb, dump.device)
    _check("moe_debug_prefill_operand", lib().moe_debug_prefill_operand(ctypes.byref(pool), int(gemm), int(slot),
                                                                        int(m0), _p(dump), _p(ws), nb,
                                                                        _stream(stream)))
    return ws


def moe_dequantize(pool: moe_pool, slot, matrix, out, stream=None):
    _check("moe_dequantize", lib().moe_dequantize(ctypes.byref(pool), slot, matrix, _p(out), _stream(stream)))


def moe_expert_hist(ids, E, counts, stream=None):
    """counts[e] += occurrences of e in ids (int32 [T][k], device); counts uint32 [E], device."""
    T, k = ids.shape
    _check("moe_expert_hist", lib().moe_expert_hist(_p(ids), T, k, E, _p(counts), _stream(stream)))


def moe_cache_plan(score, slot_table, slots, hysteresis=1.0, max_moves=None):
    """Host plan of admissions/evictions.  score float32 [E], slot_table int32 [E],
    slots int32 [n] (numpy).  Returns (moves int32 [n_moves][3] as (slot, evict,
    admit), new_slot_table int32 [E])."""
    score = np.ascontiguousarray(score, np.float32)
    table = np.ascontiguousarray(slot_table, np.int32)
    slots = np.ascontiguousarray(slots, np.int32)
    E = score.shape[0]
    if table.shape != (E,):
        raise ValueError("slot_table must have E entries")
    m = len(slots) if max_moves is None else int(max_moves)
    moves = np.zeros((max(m, 1), 3), np.int32)
    new_table = np.empty(E, np.int32)
    n = lib().moe_cache_plan(score.ctypes.data, E, table.ctypes.data, slots.ctypes.data if len(slots) else None,
                             len(slots), float(hysteresis), m, moves.ctypes.data, new_table.ctypes.data)
    if n < 0:
        raise MoeError("moe_cache_plan", n)
    return moves[:n].copy(), new_table


def moe_slot_fill(pool: moe_pool, slot, host_codes, host_scales, stream=None):
    """Copy one expert's packed weights (host uint8 tensors, pinned for overlap) into a pool slot."""
    for t in (host_codes, host_scales):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host_codes / host_scales must be contiguous host tensors")
    _check("moe_slot_fill", lib().moe_slot_fill(ctypes.byref(pool), int(slot), ctypes.c_void_p(host_codes.data_ptr()),
                                                ctypes.c_void_p(host_scales.data_ptr()), _stream(stream)))


class Layer:
    """Buffers and calls for one MoE layer at a fixed token count: the three
    C-ABI calls in order on one stream.  Buffers are allocated once here (the
    library itself never allocates)."""

    def __init__(self, pool: synth.PoolData, shared_slot, slot_table, Wr, bias, k, T, device="cuda"):
        self.pool_data = pool
        self.pool = make_pool(pool, shared_slot)
        self.slot_table, self.Wr, self.bias, self.k, self.T = slot_table, Wr, bias, k, T
        D, E = Wr.shape[1], Wr.shape[0]
        self.D, self.E = D, E
        self.ids = torch.empty(T, k, dtype=torch.int32, device=device)
        self.gates = torch.empty(T, k, dtype=torch.float32, device=device)
        self.logits = torch.empty(T, E, dtype=torch.float32, device=device)
        self.route_ws = alloc_ws(route_workspace_size(T, D, E, k), device)
        self.ws = alloc_ws(workspace_size(T, D, pool.d_ff, E, k, pool.fmt), device)
        self.expert_out = alloc_ws(expert_out_size(T, D, k), device)
        self.miss_list = torch.empty(max(T * k, 1), 3, dtype=torch.int32, device=device)
        self.miss_count = torch.zeros(1, dtype=torch.int32, device=device)
        self.out = torch.empty(T, D, dtype=torch.bfloat16, device=device)
        n = layer_workspace_size(T, D, pool.d_ff, E, k, pool.fmt)
        self.layer_ws = alloc_ws(n, device) if n else None
        self.ws_fp8 = None

    def fused(self, x, residual=None, out=None, stream=None):
        """The same layer through moe_layer_forward (T <= 8; no miss_partial)."""
        out = self.out if out is None else out
        if self.layer_ws is None:
            raise MoeError("moe_layer_forward", MOE_ERR_UNSUPPORTED)
        moe_layer_forward(self.pool, self.slot_table, x, self.Wr, self.bias, self.k, self.ids, self.gates,
                          self.expert_out, self.miss_list, self.miss_count, out, self.layer_ws, residual=residual,
                          stream=stream)
        return out

    def __call__(self, x, miss_partial=None, residual=None, out=None, stream=None, with_logits=False, fp8=False):
        """The three calls; fp8=True takes moe_expert_forward_fp8 for the expert pass."""
        out = self.out if out is None else out
        moe_route_topk(x, self.Wr, self.bias, self.k, self.ids, self.gates, self.route_ws,
                       logits=self.logits if with_logits else None, stream=stream)
        if fp8:
            if self.ws_fp8 is None:
                self.ws_fp8 = alloc_ws(workspace_size_fp8(self.T, self.D, self.pool_data.d_ff, self.E, self.k,
                                                          self.pool_data.fmt), x.device)
            moe_expert_forward_fp8(self.pool, self.slot_table, x, self.ids, self.k, self.expert_out, self.miss_list,
                                   self.miss_count, self.ws_fp8, stream=stream)
        else:
            moe_expert_forward(self.pool, self.slot_table, x, self.ids, self.k, self.expert_out, self.miss_list,
                               self.miss_count, self.ws, stream=stream)
        moe_combine(self.expert_out, self.gates, x.shape[0], self.D, self.k, out, miss_partial=miss_partial,
                    residual=residual, stream=stream)
        return out
