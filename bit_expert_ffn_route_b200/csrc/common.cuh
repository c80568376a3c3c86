// common.cuh — device helpers shared by the kernels of the expert pass.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

#define MOE_DEVINL __device__ __forceinline__

namespace moe {

constexpr int kMaxTopK = 16;
constexpr int kDecodeMaxT = 8;        // tokens per launch of the decode expert pass (tensor-core GEMV over bulk-copied codes)
constexpr int kDecodeLayoutMaxT = 24; // T <= 24: the decode expert pass (launches of up to 8 tokens) and its fp32 row layout
// The router computes logits on CUDA cores in the canonical order for T <= 8
// tokens when x (fp32) and four rows of Wr fit in its shared memory
// ((4 T + 8) D bytes <= kRouteDecodeSmem); otherwise on the tensor cores, with
// each token's candidates recomputed in the canonical order.
constexpr int kRouteDecodeMaxT = 8;
constexpr size_t kRouteDecodeSmem = 192 * 1024;

MOE_DEVINL float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }
MOE_DEVINL float bf16lo(uint32_t packed) { return __uint_as_float(packed << 16); }
MOE_DEVINL float bf16hi(uint32_t packed) { return __uint_as_float(packed & 0xffff0000u); }

// fp32 -> bf16 bits, round to nearest even (finite inputs; NaN kept quiet).
MOE_DEVINL uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

MOE_DEVINL float f16_bits_to_f32(uint32_t h) {
    return __half2float(__ushort_as_half((unsigned short)h));
}

// Magic-float decode of a code field: `word` holds the code at bit position
// p (p + width <= 23); the result is 2^(23-p) + code exactly.
template <int P, int WIDTH>
MOE_DEVINL float magic_code(uint32_t word) {
    constexpr uint32_t mask = ((1u << WIDTH) - 1u) << P;
    constexpr uint32_t expo = (uint32_t)(127 + 23 - P) << 23;
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(word), "n"(mask), "r"(expo));
    return __uint_as_float(r);   // (word & mask) | expo
}
template <int P>
constexpr float magic_base() { return (float)(1u << (23 - P)); }

MOE_DEVINL uint32_t ld_nc_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
MOE_DEVINL uint2 ld_nc_u64(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
MOE_DEVINL uint4 ld_nc_u128(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

}  // namespace moe

// Host-side launch helpers ---------------------------------------------------
namespace moe {
inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }
inline moe_status last_launch_status() { return cuda_status(cudaGetLastError()); }
}  // namespace moe
