"""The weight operand the prefill tensor cores consume, bit for bit.

moe_debug_prefill_operand runs the prefill GEMM kernel on one tile and reads
its dequantised weight operand back out of shared memory.  Every fp16 weight must
be the exact weight of the block format rounded once to fp16 (round to nearest
even): the oracle's fp32 dequantisation (exact for these pools: s*q + m and
d*(sc-32)*(q-4) need at most 17 significant bits) converted by numpy's
float32 -> float16 cast.  Covers the three formats, both GEMMs (gate|up rows
0..127 gate and 128..255 up; down rows = outputs) and first / last tiles."""
import numpy as np
import pytest
import torch

import oracle
from bit_expert_ffn_route_b200 import moe, synth

pytestmark = pytest.mark.gpu

D, F = 3072, 512


def decode_dump(dump, K):
    """uint32 [K/64][256][32] -> fp16 bit patterns [256][K] (the documented word order)."""
    R = K // 64
    d = dump.reshape(R, 256, 32)
    lo = (d & 0xFFFF).astype(np.uint16)
    hi = (d >> 16).astype(np.uint16)
    W = np.zeros((256, K), np.uint16)
    for rr in range(R):
        for j in range(32):
            c = j // 4
            k0 = 64 * rr + 16 * (c // 2) + 4 * (c % 2) + j % 4
            W[:, k0] = lo[rr, :, j]
            W[:, k0 + 8] = hi[rr, :, j]
    return W


@pytest.mark.parametrize("fmt", [synth.Q2_32, synth.Q3_32, synth.Q3_S256])
def test_prefill_operand_is_rne_fp16_of_exact_weight(fmt):
    pool = synth.make_pool(fmt, D, F, 3, seed=40 + fmt, device="cuda")
    p = moe.make_pool(pool, 0)
    host = oracle.HostPool(fmt, D, F, 3, 0, pool.codes.cpu().numpy(), pool.scales.cpu().numpy(),
                           pool.stride_codes, pool.stride_scales)
    for slot in (1, 2):
        gate, up, down = (oracle.dequant(host, slot, m) for m in range(3))
        for gemm, m0 in ((1, 0), (1, F - 128), (2, 0), (2, D - 256)):
            K = D if gemm == 1 else F
            dump = torch.zeros(K // 64 * 256 * 32, dtype=torch.int32, device="cuda")
            moe.moe_debug_prefill_operand(p, gemm, slot, m0, dump)
            torch.cuda.synchronize()
            got = decode_dump(dump.cpu().numpy().view(np.uint32), K)
            if gemm == 1:
                want32 = np.concatenate([gate[m0:m0 + 128], up[m0:m0 + 128]])
            else:
                want32 = down[m0:m0 + 256]
            want = want32.astype(np.float16).view(np.uint16)
            bad = np.argwhere(got != want)[:6]
            detail = [(int(r), int(c), float(got[r, c:c + 1].view(np.float16)[0]),
                       float(want[r, c:c + 1].view(np.float16)[0]), float(want32[r, c])) for r, c in bad]
            assert np.array_equal(got, want), (slot, gemm, m0, int((got != want).sum()), detail)
