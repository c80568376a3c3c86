"""Shared helpers of the GPU parity tests: marshalling between torch, the CUDA
binding and the oracle.  The oracle only ever receives generator outputs or
its own results; nothing the CUDA path computes is fed to it."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.uint16).cpu().numpy()


def bf16_from_u16(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16)).view(torch.bfloat16).to(device)


def f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def rel_l2_per_token(got_bits, want_bits) -> np.ndarray:
    g, w = f64(got_bits), f64(want_bits)
    return np.linalg.norm(g - w, axis=1) / np.maximum(np.linalg.norm(w, axis=1), 1e-30)


def mini_pool(pool, slots, shared_slot):
    """HostPool holding only `slots` (copied from the generator's pool), plus a
    map old slot -> new index.  shared_slot is always included."""
    want = sorted(set(int(s) for s in slots if s >= 0) | {int(shared_slot)})
    sc, ss = pool.stride_codes, pool.stride_scales
    codes = np.empty(len(want) * sc, np.uint8)
    scales = np.empty(len(want) * ss, np.uint8)
    for i, s in enumerate(want):
        c, m = pool.slot_host(s)
        codes[i * sc:(i + 1) * sc] = c
        scales[i * ss:(i + 1) * ss] = m
    remap = {s: i for i, s in enumerate(want)}
    hp = oracle.HostPool(pool.fmt, pool.d_model, pool.d_ff, len(want), remap[int(shared_slot)],
                         codes, scales, sc, ss)
    return hp, remap


def oracle_layer(pool, layer, k, x_bits, miss_partial=None, residual_bits=None, n_threads=8, fp8=False):
    """The oracle's full expert pass for the tokens x_bits, reading only the
    slots it needs from the generated pool (fp8: its e4m3-operand variant)."""
    Wr = u16(layer.Wr)
    bias = None if layer.bias is None else layer.bias.detach().float().cpu().numpy()
    table = layer.slot_table.detach().cpu().numpy().astype(np.int32)
    ids, _ = oracle.topk_gates(oracle.router_logits(x_bits, Wr, bias), k)
    sel = np.unique(ids)
    hp, remap = mini_pool(pool, [table[e] for e in sel if 0 <= table[e] < pool.n_slots], layer.shared_slot)
    mini_table = np.full_like(table, -1)
    for e in sel:
        s = int(table[e])
        if 0 <= s < pool.n_slots:
            mini_table[e] = remap[s]
    return oracle.moe_layer(hp, mini_table, k, x_bits, Wr, bias, miss_partial=miss_partial,
                            residual=residual_bits, n_threads=n_threads, fp8=fp8)
