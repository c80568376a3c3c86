// hooks.cu — test hooks of the C ABI: the exact dequantiser of one matrix and
// a bounded wait on a device flag (for testing the device error word).
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

namespace moe {
namespace {

// Test hook: one thread per block of one row; exact fp32 weights.
__global__ void dequant_kernel(PoolView P, int slot, int mat, float* __restrict__ out) {
    const int rows = (mat == 2) ? P.D : P.F;
    const int K = (mat == 2) ? P.F : P.D;
    const int bw = (P.fmt == MOE_Q3_S256) ? 256 : 32;
    const int nbk = K / bw;
    const size_t blocks = (size_t)P.D * P.F / bw;
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= rows * nbk) return;
    const int row = idx / nbk, b = idx % nbk;
    const uint8_t* codes = P.codes + (size_t)slot * P.stride_c;
    const uint8_t* meta = P.scales + (size_t)slot * P.stride_s;
    float* o = out + (size_t)row * K + (size_t)b * bw;
    if (P.fmt == MOE_Q3_S256) {
        const uint8_t* c = codes + ((size_t)mat * blocks + (size_t)row * nbk + b) * 96;
        const uint8_t* sc = meta + ((size_t)mat * blocks + (size_t)row * nbk + b) * 12;
        const uint16_t dbits = *reinterpret_cast<const uint16_t*>(meta + 3 * blocks * 12 +
                                                                 ((size_t)mat * blocks + (size_t)row * nbk + b) * 2);
        const float d = f16_bits_to_f32(dbits);
        for (int i = 0; i < 256; ++i) {
            const int bit = 3 * i;
            const uint32_t two = (uint32_t)c[bit >> 3] | ((uint32_t)((bit >> 3) + 1 < 96 ? c[(bit >> 3) + 1] : 0) << 8);
            const int q = (two >> (bit & 7)) & 7;
            const int sbit = 6 * (i >> 4);
            const uint32_t stwo = (uint32_t)sc[sbit >> 3] | ((uint32_t)((sbit >> 3) + 1 < 12 ? sc[(sbit >> 3) + 1] : 0) << 8);
            const int s6 = (stwo >> (sbit & 7)) & 63;
            o[i] = d * (float)((s6 - 32) * (q - 4));   // integer product first: exact, +0.0 for q == 4
        }
    } else {
        const int nbits = (P.fmt == MOE_Q2_32) ? 2 : 3;
        const int cb = (P.fmt == MOE_Q2_32) ? 8 : 12;
        const uint8_t* c = codes + ((size_t)mat * blocks + (size_t)row * nbk + b) * cb;
        const uint32_t sm = *reinterpret_cast<const uint32_t*>(meta + ((size_t)mat * blocks + (size_t)row * nbk + b) * 4);
        const float s = f16_bits_to_f32(sm & 0xffffu), m = f16_bits_to_f32(sm >> 16);
        for (int j = 0; j < 32; ++j) {
            const int bit = nbits * j;
            const uint32_t two = (uint32_t)c[bit >> 3] | ((uint32_t)((bit >> 3) + 1 < cb ? c[(bit >> 3) + 1] : 0) << 8);
            const int q = (two >> (bit & 7)) & ((1 << nbits) - 1);
            o[j] = __fmaf_rn(s, (float)q, m);
        }
    }
}

// One thread polls *flag (acquire, gpu scope) until it equals `expect` or
// limit_ns has passed; on the limit it sets the timeout bit of *err.  A wait
// that finds the timeout bit already set returns at once.
__global__ void wait_flag_kernel(const uint32_t* flag, uint32_t expect, uint64_t limit_ns, uint32_t* err) {
    if (timed_out(err)) return;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v == expect) return;
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(err, kErrTimeout);
            return;
        }
        __nanosleep(1000);
    }
}

}  // namespace

moe_status launch_dequantize(const PoolView& P, int slot, int matrix, float* out, cudaStream_t s) {
    const int rows = (matrix == 2) ? P.D : P.F;
    const int K = (matrix == 2) ? P.F : P.D;
    const int bw = (P.fmt == MOE_Q3_S256) ? 256 : 32;
    const int n = rows * (K / bw);
    dequant_kernel<<<(n + 127) / 128, 128, 0, s>>>(P, slot, matrix, out);
    return last_launch_status();
}

moe_status launch_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t limit_us, uint32_t* err, cudaStream_t s) {
    wait_flag_kernel<<<1, 1, 0, s>>>(flag, expect, (uint64_t)limit_us * 1000ull, err);
    return last_launch_status();
}

}  // namespace moe
