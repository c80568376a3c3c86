"""Seeded synthetic inputs for the routed-MoE expert pass.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's callers.  It draws random numbers and lays them out in the pool's byte
format; it holds none of the method's arithmetic (no routing, no dequantisation,
no FFN).  The pages publish no weights or value distributions, so the recipe is
ours and is stated here:

* hidden states: bf16 of N(0, 1);
* router weights ``Wr``: bf16 of N(0, 0.02);
* router bias (optional): ``b[e] = -alpha * s * ln(rank(e))`` where ``rank`` is a
  seeded permutation of 1..E (a Zipf(s) popularity prior, strength ``alpha``);
* weights of zero mean and standard deviation ~``weight_std`` (default 0.02):
* Q2_32 / Q3_32 codes: uniform random bytes (so every code is uniform);
  ``s = fp16(c * (0.5 + U))`` with ``c = weight_std / sqrt(1.25)`` (Q2, codes 0..3)
  or ``weight_std / sqrt(5.25)`` (Q3, codes 0..7); ``m = fp16(-1.5 s)`` (Q2) or
  ``fp16(-3.5 s)`` (Q3), centring the codes;
* Q3_S256 codes and 6-bit sub-scales: uniform random bytes;
  ``d = fp16(weight_std / 43.3 * (0.5 + U))`` (43.3 = rms of (sc - 32)(q - 4)).

Layout of one slot (bytes, each region 256-byte padded):
  codes : gate plane [F][D/bw][cb] | up plane [F][D/bw][cb] | down plane [D][F/bw][cb]
  scales: Q2/Q3_32: (s, m) fp16 pairs, planes in the same order;
          Q3_S256: 12-byte sub-scale planes (gate, up, down) then fp16 d planes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

Q2_32, Q3_32, Q3_S256 = 0, 1, 2
FMT_NAMES = {Q2_32: "q2_32", Q3_32: "q3_32", Q3_S256: "q3_s256"}

_BLOCK = {Q2_32: 32, Q3_32: 32, Q3_S256: 256}
_CODE_BYTES = {Q2_32: 8, Q3_32: 12, Q3_S256: 96}


def _round_up(n: int, a: int) -> int:
    return (n + a - 1) // a * a


def slot_code_bytes(fmt: int, D: int, F: int) -> int:
    return 3 * D * F // _BLOCK[fmt] * _CODE_BYTES[fmt]


def slot_scale_bytes(fmt: int, D: int, F: int) -> int:
    n = 3 * D * F // _BLOCK[fmt]
    return n * (14 if fmt == Q3_S256 else 4)


def generator(seed: int, *stream: int, device="cpu") -> torch.Generator:
    """A torch generator for the sub-stream (seed, *stream)."""
    state = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, *[int(s) & 0xFFFFFFFF for s in stream]])
    g = torch.Generator(device=device)
    g.manual_seed(int(state.generate_state(1, np.uint64)[0] >> np.uint64(1)))
    return g


def hidden(T: int, D: int, seed: int, stream: int = 0, device="cpu") -> torch.Tensor:
    g = generator(seed, 1, stream)
    return torch.randn(T, D, generator=g, dtype=torch.float32).to(torch.bfloat16).to(device)


def router_weight(E: int, D: int, seed: int, layer: int = 0, device="cpu") -> torch.Tensor:
    g = generator(seed, 2, layer)
    return (torch.randn(E, D, generator=g, dtype=torch.float32) * 0.02).to(torch.bfloat16).to(device)


def popularity_order(E: int, seed: int, layer: int = 0) -> torch.Tensor:
    """order[i] = the expert whose popularity rank is i + 1 (rank 1 = most popular)."""
    g = generator(seed, 3, layer)
    return torch.randperm(E, generator=g)


def zipf_bias(E: int, s: float, alpha: float, seed: int, layer: int = 0) -> torch.Tensor:
    """fp32 bias b[order[i]] = -alpha * s * ln(i + 1)."""
    order = popularity_order(E, seed, layer)
    b = torch.empty(E, dtype=torch.float64)
    b[order] = -alpha * s * torch.log(torch.arange(1, E + 1, dtype=torch.float64))
    return b.to(torch.float32)


def slot_table(E: int, resident: torch.Tensor, slots: torch.Tensor) -> torch.Tensor:
    """int32 [E]: slot_table[resident[i]] = slots[i]; every other expert -> -1."""
    t = torch.full((E,), -1, dtype=torch.int32)
    t[resident.long()] = slots.to(torch.int32)
    return t


def slot_permutation(n: int, seed: int, stream: int = 0) -> torch.Tensor:
    g = generator(seed, 4, stream)
    return torch.randperm(n, generator=g)


@dataclass
class PoolData:
    """A quantised expert pool: ``codes``/``scales`` are flat uint8 tensors."""
    fmt: int
    d_model: int
    d_ff: int
    n_slots: int
    codes: torch.Tensor
    scales: torch.Tensor
    stride_codes: int
    stride_scales: int

    @property
    def slot_bytes(self) -> int:
        return slot_code_bytes(self.fmt, self.d_model, self.d_ff) + slot_scale_bytes(self.fmt, self.d_model, self.d_ff)

    def slot_host(self, slot: int):
        """(codes, scales) bytes of one slot as numpy arrays."""
        c = self.codes[slot * self.stride_codes:(slot + 1) * self.stride_codes].cpu().numpy()
        s = self.scales[slot * self.stride_scales:(slot + 1) * self.stride_scales].cpu().numpy()
        return c, s


def _random_bytes(n: int, g: torch.Generator, device) -> torch.Tensor:
    return torch.randint(0, 256, (n,), generator=g, dtype=torch.uint8, device=device)


def make_pool(fmt: int, D: int, F: int, n_slots: int, seed: int, device="cpu",
              pool_id: int = 0, chunk_slots: int = 512, weight_std: float = 0.02) -> PoolData:
    """Generate ``n_slots`` experts in the pool format (see module docstring)."""
    cb = slot_code_bytes(fmt, D, F)
    sb = slot_scale_bytes(fmt, D, F)
    stride_c, stride_s = _round_up(cb, 256), _round_up(sb, 256)
    codes = torch.zeros(n_slots * stride_c, dtype=torch.uint8, device=device)
    scales = torch.zeros(n_slots * stride_s, dtype=torch.uint8, device=device)
    cv = codes.view(n_slots, stride_c)
    sv = scales.view(n_slots, stride_s)
    n_blocks = 3 * D * F // _BLOCK[fmt]
    for c0 in range(0, n_slots, chunk_slots):
        c1 = min(n_slots, c0 + chunk_slots)
        n = c1 - c0
        g = generator(seed, 5, pool_id, c0, device=device)
        cv[c0:c1, :cb] = _random_bytes(n * cb, g, device).view(n, cb)
        u = torch.rand(n, n_blocks, generator=g, device=device, dtype=torch.float32)
        if fmt == Q3_S256:
            sc = _random_bytes(n * n_blocks * 12, g, device).view(n, n_blocks * 12)
            d = (weight_std / 43.3 * (0.5 + u)).to(torch.float16)
            sv[c0:c1, :n_blocks * 12] = sc
            sv[c0:c1, n_blocks * 12:n_blocks * 14] = d.view(torch.uint8).view(n, n_blocks * 2)
        else:
            c = weight_std / (1.25 ** 0.5 if fmt == Q2_32 else 5.25 ** 0.5)
            s = (c * (0.5 + u)).to(torch.float16)
            m = (-(1.5 if fmt == Q2_32 else 3.5) * s.float()).to(torch.float16)
            sm = torch.stack([s, m], dim=-1)            # s at the lower address
            sv[c0:c1, :sb] = sm.view(torch.uint8).view(n, sb)
    return PoolData(fmt, D, F, n_slots, codes, scales, stride_c, stride_s)
