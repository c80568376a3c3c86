"""Test-side statement of the block formats: packs chosen codes and scales into
pool bytes with plain Python integers, independently of the oracle's C
unpacker, of the CUDA kernels and of the synthetic generator.

Format (a reading; the pages name Q2_0 / IQ3_S-class formats of ~2-3.5 bits per
weight without defining them): per slot, code planes gate [F][D/bw], up [F][D/bw],
down [D][F/bw] (row-major, blocks along the reduction dimension); each block's
codes form a little-endian bit stream, weight j at bits [nbits*j, nbits*(j+1)).
Meta: Q2/Q3_32 an (s, m) fp16 pair per block, s first; Q3_S256 a 12-byte 6-bit
sub-scale stream per super-block (sub-block j at bits [6j, 6j+6)), all three
matrices' sub-scale planes first, then their fp16 d planes.
"""
from __future__ import annotations

import numpy as np

Q2_32, Q3_32, Q3_S256 = 0, 1, 2
BW = {Q2_32: 32, Q3_32: 32, Q3_S256: 256}
NBITS = {Q2_32: 2, Q3_32: 3, Q3_S256: 3}
CB = {Q2_32: 8, Q3_32: 12, Q3_S256: 96}


def pack_stream(values, nbits, nbytes):
    acc = 0
    for j, v in enumerate(values):
        assert 0 <= int(v) < (1 << nbits)
        acc |= int(v) << (nbits * j)
    return list(acc.to_bytes(nbytes, "little"))


def f16_bits(v):
    return int(np.array([v], dtype=np.float16).view(np.uint16)[0])


def shapes(D, F):
    return [(F, D), (F, D), (D, F)]          # gate, up, down: (rows, K)


class SlotBuilder:
    """Builds the bytes of one slot from per-matrix integer codes and block meta."""

    def __init__(self, fmt, D, F):
        self.fmt, self.D, self.F = fmt, D, F
        self.codes = [np.zeros(s, np.int64) for s in shapes(D, F)]
        bw = BW[fmt]
        if fmt == Q3_S256:
            self.sub = [np.full((r, K // bw, 16), 32, np.int64) for r, K in shapes(D, F)]
            self.d = [np.zeros((r, K // bw), np.float16) for r, K in shapes(D, F)]
        else:
            self.s = [np.zeros((r, K // bw), np.float16) for r, K in shapes(D, F)]
            self.m = [np.zeros((r, K // bw), np.float16) for r, K in shapes(D, F)]

    def code_bytes(self):
        out = []
        bw, nb, cb = BW[self.fmt], NBITS[self.fmt], CB[self.fmt]
        for mat, (rows, K) in zip(self.codes, shapes(self.D, self.F)):
            for r in range(rows):
                for b in range(K // bw):
                    out += pack_stream(mat[r, b * bw:(b + 1) * bw], nb, cb)
        return np.array(out, np.uint8)

    def scale_bytes(self):
        out = []
        if self.fmt == Q3_S256:
            for sub in self.sub:
                for r in range(sub.shape[0]):
                    for b in range(sub.shape[1]):
                        out += pack_stream(sub[r, b], 6, 12)
            for d in self.d:
                for v in d.ravel():
                    out += list(int(np.array([v], np.float16).view(np.uint16)[0]).to_bytes(2, "little"))
        else:
            for s, m in zip(self.s, self.m):
                for sv, mv in zip(s.ravel(), m.ravel()):
                    out += list(f16_bits(sv).to_bytes(2, "little"))
                    out += list(f16_bits(mv).to_bytes(2, "little"))
        return np.array(out, np.uint8)

    def weights(self):
        """The exact weights these codes and scales stand for (float64 matrices)."""
        bw = BW[self.fmt]
        res = []
        for i, (rows, K) in enumerate(shapes(self.D, self.F)):
            q = self.codes[i].astype(np.float64)
            if self.fmt == Q3_S256:
                sub = np.repeat(self.sub[i], 16, axis=2).reshape(rows, K).astype(np.float64)
                d = np.repeat(self.d[i].astype(np.float64), bw, axis=1)
                res.append(d * (sub - 32) * (q - 4))
            else:
                s = np.repeat(self.s[i].astype(np.float64), bw, axis=1)
                m = np.repeat(self.m[i].astype(np.float64), bw, axis=1)
                res.append(s * q + m)
        return res


def build_pool(builders, shared_slot=0):
    """HostPool (oracle) from SlotBuilders, slot strides padded to 256 bytes."""
    import oracle
    b0 = builders[0]
    cbytes = [b.code_bytes() for b in builders]
    sbytes = [b.scale_bytes() for b in builders]
    sc = -(-len(cbytes[0]) // 256) * 256
    ss = -(-len(sbytes[0]) // 256) * 256
    codes = np.zeros(sc * len(builders), np.uint8)
    scales = np.zeros(ss * len(builders), np.uint8)
    for i, (c, s) in enumerate(zip(cbytes, sbytes)):
        codes[i * sc:i * sc + len(c)] = c
        scales[i * ss:i * ss + len(s)] = s
    return oracle.HostPool(b0.fmt, b0.D, b0.F, len(builders), shared_slot, codes, scales, sc, ss)
