"""CPU oracle of the routed-MoE expert pass (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``liboracle.so`` (plain C,
built from ``moe_oracle.c`` by :func:`build`) with numpy arrays; it shares no
code with the CUDA library and never calls it.

Every array crossing this boundary is a numpy array on the host:
bf16 values travel as their ``uint16`` bit patterns, fp16 likewise.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

Q2_32, Q3_32, Q3_S256 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (OpenMP) if it is missing or stale."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                                   os.path.getmtime(os.path.join(_HERE, "moe_oracle.h"))))
    if force or stale:
        # -ffp-contract=off: no fused multiply-add unless the source asks for fmaf.
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


class _Pool(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("n_slots", ctypes.c_int), ("shared_slot", ctypes.c_int),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("stride_codes", ctypes.c_size_t), ("stride_scales", ctypes.c_size_t)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.orc_slot_code_bytes.restype = ctypes.c_size_t
        L.orc_slot_code_bytes.argtypes = [i, i, i]
        L.orc_slot_scale_bytes.restype = ctypes.c_size_t
        L.orc_slot_scale_bytes.argtypes = [i, i, i]
        L.orc_router_logits.argtypes = [P, i, i, P, P, i, P]
        L.orc_topk_gates.argtypes = [P, i, i, i, P, P]
        L.orc_slot_lookup.argtypes = [P, i, i, P, i, i, P, P]
        L.orc_dequant.argtypes = [ctypes.POINTER(_Pool), i, i, P]
        L.orc_expert.argtypes = [ctypes.POINTER(_Pool), i, P, P, P]
        L.orc_moe_layer.argtypes = [ctypes.POINTER(_Pool), P, i, i, P, i, P, P, P, P,
                                    P, P, P, P, P, P, i]
        L.orc_moe_layer_fp8.argtypes = L.orc_moe_layer.argtypes
        L.orc_expert_fp8.argtypes = [ctypes.POINTER(_Pool), i, P, P]
        L.orc_e4m3_rne.restype = ctypes.c_uint8
        L.orc_e4m3_rne.argtypes = [ctypes.c_double]
        L.orc_e4m3_to_f64.restype = ctypes.c_double
        L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_f16_round.restype = ctypes.c_double
        L.orc_f16_round.argtypes = [ctypes.c_double]
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_bf16_rne.argtypes = [ctypes.c_double]
        L.orc_f16_to_f32.restype = ctypes.c_float
        L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


@dataclass
class HostPool:
    """A quantised expert pool held in host memory (bytes exactly as on the device)."""
    fmt: int
    d_model: int
    d_ff: int
    n_slots: int
    shared_slot: int
    codes: np.ndarray      # uint8 [n_slots * stride_codes]
    scales: np.ndarray     # uint8 [n_slots * stride_scales]
    stride_codes: int
    stride_scales: int

    def _c(self):
        self.codes = np.ascontiguousarray(self.codes, dtype=np.uint8)
        self.scales = np.ascontiguousarray(self.scales, dtype=np.uint8)
        return _Pool(self.fmt, self.d_model, self.d_ff, self.n_slots, self.shared_slot,
                     self.codes.ctypes.data, self.scales.ctypes.data,
                     self.stride_codes, self.stride_scales)


def slot_code_bytes(fmt, D, F):
    return int(lib().orc_slot_code_bytes(fmt, D, F))


def slot_scale_bytes(fmt, D, F):
    return int(lib().orc_slot_scale_bytes(fmt, D, F))


def router_logits(x, Wr, bias=None):
    x = _c(x, np.uint16); Wr = _c(Wr, np.uint16); bias = _c(bias, np.float32)
    T, D = x.shape
    E = Wr.shape[0]
    out = np.empty((T, E), np.float32)
    rc = lib().orc_router_logits(_ptr(x), T, D, _ptr(Wr), _ptr(bias), E, _ptr(out))
    if rc != 0:
        raise ValueError("orc_router_logits: bad arguments")
    return out


def topk_gates(logits, k):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float64)
    if lib().orc_topk_gates(_ptr(logits), T, E, k, _ptr(ids), _ptr(gates)) != 0:
        raise ValueError("orc_topk_gates: bad arguments")
    return ids, gates


def slot_lookup(ids, slot_table, n_slots):
    ids = _c(ids, np.int32); st = _c(slot_table, np.int32)
    T, k = ids.shape
    slots = np.empty((T, k), np.int32)
    miss = np.empty((max(T * k, 1), 3), np.int32)
    n = lib().orc_slot_lookup(_ptr(ids), T, k, _ptr(st), st.shape[0], n_slots, _ptr(slots), _ptr(miss))
    if n < 0:
        raise ValueError("orc_slot_lookup: bad arguments")
    return slots, miss[:n].copy()


def dequant(pool: HostPool, slot: int, matrix: int) -> np.ndarray:
    D, F = pool.d_model, pool.d_ff
    shape = (D, F) if matrix == 2 else (F, D)
    out = np.empty(shape, np.float32)
    p = pool._c()
    if lib().orc_dequant(ctypes.byref(p), slot, matrix, _ptr(out)) != 0:
        raise ValueError("orc_dequant: bad arguments")
    return out


def expert(pool: HostPool, slot: int, x):
    """One expert on one token: returns (h bf16 bits [F], y float64 [D])."""
    x = _c(x, np.uint16)
    h = np.empty(pool.d_ff, np.uint16)
    y = np.empty(pool.d_model, np.float64)
    p = pool._c()
    if lib().orc_expert(ctypes.byref(p), slot, _ptr(x), _ptr(h), _ptr(y)) != 0:
        raise ValueError("orc_expert: bad arguments")
    return h, y


@dataclass
class LayerResult:
    out: np.ndarray        # uint16 (bf16 bits) [T, D]
    logits: np.ndarray     # float32 [T, E]
    ids: np.ndarray        # int32 [T, k]
    gates: np.ndarray      # float64 [T, k]
    slots: np.ndarray      # int32 [T, k]
    miss_list: np.ndarray  # int32 [n_miss, 3]


def moe_layer(pool: HostPool, slot_table, k, x, Wr, bias=None, miss_partial=None,
              residual=None, n_threads: int = 1, fp8: bool = False) -> LayerResult:
    """The whole expert pass for T tokens (see moe_oracle.h); fp8=True is the
    e4m3-operand variant (orc_moe_layer_fp8)."""
    x = _c(x, np.uint16); Wr = _c(Wr, np.uint16); bias = _c(bias, np.float32)
    st = _c(slot_table, np.int32)
    mp = _c(miss_partial, np.float32); res = _c(residual, np.uint16)
    T, D = x.shape
    E = Wr.shape[0]
    out = np.empty((T, D), np.uint16)
    logits = np.empty((T, E), np.float32)
    ids = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float64)
    slots = np.empty((T, k), np.int32)
    miss = np.empty((max(T * k, 1), 3), np.int32)
    p = pool._c()
    fn = lib().orc_moe_layer_fp8 if fp8 else lib().orc_moe_layer
    n = fn(ctypes.byref(p), _ptr(st), E, k, _ptr(x), T, _ptr(Wr), _ptr(bias),
                            _ptr(mp), _ptr(res), _ptr(out), _ptr(logits), _ptr(ids), _ptr(gates),
                            _ptr(slots), _ptr(miss), int(n_threads))
    if n < 0:
        raise ValueError("orc_moe_layer: bad arguments")
    return LayerResult(out, logits, ids, gates, slots, miss[:n].copy())


def bf16_rne(v: float) -> int:
    return int(lib().orc_bf16_rne(float(v)))


def f16_to_f32(h: int) -> float:
    return float(lib().orc_f16_to_f32(int(h)))


def e4m3_rne(v: float) -> int:
    """The e4m3 byte nearest to v (ties to even, saturating at +-448)."""
    return int(lib().orc_e4m3_rne(float(v)))


def e4m3_to_f64(b: int) -> float:
    return float(lib().orc_e4m3_to_f64(int(b)))


def f16_round(v: float) -> float:
    return float(lib().orc_f16_round(float(v)))


def expert_fp8(pool: HostPool, slot: int, x):
    """The e4m3-operand variant of one expert on one token: y float64 [D]."""
    x = _c(x, np.uint16)
    y = np.empty(pool.d_model, np.float64)
    p = pool._c()
    if lib().orc_expert_fp8(ctypes.byref(p), slot, _ptr(x), _ptr(y)) != 0:
        raise ValueError("orc_expert_fp8: bad arguments")
    return y
