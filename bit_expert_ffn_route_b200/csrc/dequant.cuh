// dequant.cuh — 2-/3-bit codes to fp16 weight pairs, shared by the decode
// (mma.sync) and prefill (tcgen05) expert passes.
//
// Block formats (readings; the pages name Q2_0 and IQ3-class ~3.44 bpw
// formats without defining them: wiselychen RTX 5090 report §1 "低位元量化",
// greenbean-ai "Strata 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next" §四):
//   Q2_32 / Q3_32   w = s*q + m, q the 2-/3-bit code of the weight
//   Q3_S256         w = d*(sc - 32)*(q - 4), sc the 6-bit sub-scale of its 16
// Every fp16 weight produced here is the exact weight rounded once to fp16
// (round to nearest even):
//   Q2_32 / Q3_32   fma.rn.f16x2(s, q, m): s*q + m is formed exactly and
//                   rounded once;
//   Q3_S256         n = (sc - 32) * (q - 4) is an integer in [-128, 124],
//                   exact in fp16 (fma.rn.f16x2(sc - 32, q - 4, +0): the +0
//                   addend turns a -0 product into +0, as the integer product
//                   is), then w = mul.rn.f16x2(d, n): d * n rounded once.
//
// Code extraction: an fp16 "magic number" 2^(10-b) OR-ed with a code field
// that sits at bit b of a half gives 2^(10-b) + code exactly; subtracting the
// magic number again leaves the code (a small exact integer).  One 32-bit
// word of codes yields the weight pairs (i, i + 8) of a 16-weight group: the
// two halves of the word hold the codes of weights i and i + 8 at the same
// bit offset.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#define MOE_DEVINL __device__ __forceinline__

namespace moe {

// A value the compiler cannot fold into an immediate (lop3 takes one
// immediate; two would cost a second logic op per code).
MOE_DEVINL uint32_t opaque_u32(uint32_t v) {
    uint32_t r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}
template <uint32_t MASK>
MOE_DEVINL uint32_t field_or(uint32_t w, uint32_t magic) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "n"(MASK), "r"(magic));   // (w & MASK) | magic
    return r;
}
MOE_DEVINL uint32_t hsub2u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
MOE_DEVINL uint32_t hfma2u(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}
MOE_DEVINL uint32_t hmul2u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// Two fp32 values to f16x2 (lo in the low half), round to nearest even.
MOE_DEVINL uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// fp16 magic numbers in both halves (2^(10-b) for a field at bit b), and the
// same plus 4 (the Q3_S256 code centre) for the centred 3-bit fields.
struct Magic {
    uint32_t m1024, m256, m128, m64, m16, m8, m4;
    uint32_t s1028, s132, s20, s12;
};
MOE_DEVINL Magic make_magic() {
    Magic m;
    m.m1024 = opaque_u32(0x64006400u);
    m.m256 = opaque_u32(0x5C005C00u);
    m.m128 = opaque_u32(0x58005800u);
    m.m64 = opaque_u32(0x54005400u);
    m.m16 = opaque_u32(0x4C004C00u);
    m.m8 = opaque_u32(0x48004800u);
    m.m4 = opaque_u32(0x44004400u);
    m.s1028 = opaque_u32(0x64046404u);
    m.s132 = opaque_u32(0x58205820u);
    m.s20 = opaque_u32(0x4D004D00u);
    m.s12 = opaque_u32(0x4A004A00u);
    return m;
}

// ---------------------------------------------------------------- Q2: 16 codes per word
// Word w holds code i of a 16-weight group at bits [2i, 2i+2); w10 = w >> 10.
// q2_codes<F>: the code pair (F, F + 8) as exact fp16 integers.
template <int F>
MOE_DEVINL uint32_t q2_codes(uint32_t w, uint32_t w10, const Magic& M) {
    if constexpr (F == 0) return hsub2u(field_or<0x00030003u>(w, M.m1024), M.m1024);
    else if constexpr (F == 1) return hsub2u(field_or<0x000C000Cu>(w, M.m256), M.m256);
    else if constexpr (F == 2) return hsub2u(field_or<0x00300030u>(w, M.m64), M.m64);
    else if constexpr (F == 3) return hsub2u(field_or<0x00C000C0u>(w, M.m16), M.m16);
    else if constexpr (F == 4) return hsub2u(field_or<0x03000300u>(w, M.m4), M.m4);
    else if constexpr (F == 5) return hsub2u(field_or<0x00030003u>(w10, M.m1024), M.m1024);
    else if constexpr (F == 6) return hsub2u(field_or<0x000C000Cu>(w10, M.m256), M.m256);
    else return hsub2u(field_or<0x00300030u>(w10, M.m64), M.m64);
}

// ---------------------------------------------------------------- Q3: 16 codes per 48 bits
// A 16-weight group of 3-bit codes is 48 stream bits.  P = (group bits [0,16) |
// [24,40)) and P2 = (bits [8,24) | [32,48)): code i of the low half (code i + 8
// of the high half) sits at bit 3i of P for i <= 4 and at bit 3i - 8 of P2 for
// i >= 5.  q3_codes<F, CENTRED>: the code pair (F, F + 8), minus 4 when CENTRED.
template <int F, bool CENTRED>
MOE_DEVINL uint32_t q3_codes(uint32_t P, uint32_t P9, uint32_t P2, uint32_t P10, const Magic& M) {
    if constexpr (F == 0) return hsub2u(field_or<0x00070007u>(P, M.m1024), CENTRED ? M.s1028 : M.m1024);
    else if constexpr (F == 1) return hsub2u(field_or<0x00380038u>(P, M.m128), CENTRED ? M.s132 : M.m128);
    else if constexpr (F == 2) return hsub2u(field_or<0x01C001C0u>(P, M.m16), CENTRED ? M.s20 : M.m16);
    else if constexpr (F == 3) return hsub2u(field_or<0x00070007u>(P9, M.m1024), CENTRED ? M.s1028 : M.m1024);
    else if constexpr (F == 4) return hsub2u(field_or<0x00380038u>(P9, M.m128), CENTRED ? M.s132 : M.m128);
    else if constexpr (F == 5) return hsub2u(field_or<0x03800380u>(P2, M.m8), CENTRED ? M.s12 : M.m8);
    else if constexpr (F == 6) return hsub2u(field_or<0x00070007u>(P10, M.m1024), CENTRED ? M.s1028 : M.m1024);
    else return hsub2u(field_or<0x00380038u>(P10, M.m128), CENTRED ? M.s132 : M.m128);
}
// The (P, P2) words of group h (0: stream bytes 0..5, 1: bytes 6..11) of a
// 32-weight block held in words c0, c1, c2 (12 code bytes).
MOE_DEVINL void q3_group_words(uint32_t c0, uint32_t c1, uint32_t c2, int h, uint32_t& P, uint32_t& P2) {
    if (h == 0) {
        P = __byte_perm(c0, c1, 0x4310);
        P2 = __byte_perm(c0, c1, 0x5421);
    } else {
        P = __byte_perm(c1, c2, 0x6532);
        P2 = __byte_perm(c1, c2, 0x7643);
    }
}

// ---------------------------------------------------------------- scales
// (s, m) fp16 pair word (s in the low half) -> s and m broadcast to f16x2.
MOE_DEVINL uint32_t bcast_lo(uint32_t sm) { return __byte_perm(sm, 0, 0x1010); }
MOE_DEVINL uint32_t bcast_hi(uint32_t sm) { return __byte_perm(sm, 0, 0x3232); }

// Q3_S256: the sub-block's signed sub-scale sc - 32 (an exact fp16 integer)
// broadcast to f16x2.
MOE_DEVINL uint32_t s256_sub(uint32_t sc6) {
    const uint32_t b = (uint32_t)__half_as_ushort(__int2half_rn((int)sc6 - 32));
    return b | (b << 16);
}
// Weight pair from the code pair q (exact fp16 integers) and the block scales.
MOE_DEVINL uint32_t w_sm(uint32_t q, uint32_t s2, uint32_t m2) { return hfma2u(s2, q, m2); }
// Q3_S256: qc = q - 4 (exact), sc2 = sc - 32 (exact), d2 = d: w = d * (sc2 * qc).
MOE_DEVINL uint32_t w_s256(uint32_t qc, uint32_t sc2, uint32_t d2) { return hmul2u(d2, hfma2u(sc2, qc, 0u)); }

}  // namespace moe
