// route_warp.cuh — warp-level router pieces shared by the decode and prefill
// routers: logits in the canonical fp32 order and the top-k selection.
#pragma once

#include "common.cuh"

namespace moe {

// Canonical logits of expert e for NT tokens whose bf16 rows are xrow[t]
// (shared or global memory).  Lane L accumulates elements 256c + 8L + j.
template <int NT>
__device__ __forceinline__ void canon_logits_warp(const uint16_t* const (&xrow)[NT], int nt, int D,
                                                  const uint16_t* __restrict__ Wr, const float* __restrict__ bias,
                                                  int E, int e, float* __restrict__ lout /* + t*E */) {
    const int lane = threadIdx.x & 31;
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
    const uint16_t* wrow = Wr + (size_t)e * D + 8 * lane;
    const int nc = D >> 8;
#pragma unroll 6
    for (int c = 0; c < nc; ++c) {
        const uint4 w = ld_nc_u128(wrow + 256 * c);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < nt) {
                const uint4 xv4 = *reinterpret_cast<const uint4*>(xrow[t] + 256 * c + 8 * lane);
                const uint32_t xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {   // element j = 2q (low half), 2q+1 (high half)
                    acc[t] = __fmaf_rn(bf16lo(xv[q]), bf16lo(wv[q]), acc[t]);
                    acc[t] = __fmaf_rn(bf16hi(xv[q]), bf16hi(wv[q]), acc[t]);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            acc[t] = __fadd_rn(acc[t], __shfl_xor_sync(0xffffffffu, acc[t], off));
    }
    if (lane == 0) {
        const float b = bias ? bias[e] : 0.0f;
#pragma unroll
        for (int t = 0; t < NT; ++t)
            if (t < nt) lout[(size_t)t * E + e] = bias ? __fadd_rn(acc[t], b) : acc[t];
    }
}

// Position of element d of a token row in the fp32 staging layout of the
// decode router: within each 256-element span, elements j = 0..3 of lane L's
// eight sit at 4L + j and elements j = 4..7 at 128 + 4L + (j - 4), so each of a
// lane's two 16-byte reads is one contiguous 512-byte sweep of the warp.
__device__ __forceinline__ int canon_stage_pos(int d) {
    const int c = d >> 8, L = (d >> 3) & 31, j = d & 7;
    return (c << 8) + ((j >> 2) << 7) + (L << 2) + (j & 3);
}

// canon_logits_warp for token rows staged in shared memory as fp32 (exact
// copies of the bf16 values) in the canon_stage_pos layout; the expert's Wr
// row comes in as wpre[c] for c < NPRE (loaded by the caller, possibly before
// waiting on the producer of x) and from global memory beyond.
template <int NT, int NPRE>
__device__ __forceinline__ void canon_logits_warp_staged(const float* __restrict__ xs /* [NT][D] */, int nt, int D,
                                                         const uint4 (&wpre)[NPRE], const uint16_t* __restrict__ Wr,
                                                         const float* __restrict__ bias, int E, int e,
                                                         float* __restrict__ lout /* + t*E */) {
    const int lane = threadIdx.x & 31;
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
    const int nc = D >> 8;
    auto span = [&](const uint4& w, int c) {
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        float wf[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) { wf[2 * q] = bf16lo(wv[q]); wf[2 * q + 1] = bf16hi(wv[q]); }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < nt) {
                const float* xr = xs + (size_t)t * D + 256 * c + 4 * lane;
                const float4 a = *reinterpret_cast<const float4*>(xr);
                const float4 b = *reinterpret_cast<const float4*>(xr + 128);
                acc[t] = __fmaf_rn(a.x, wf[0], acc[t]);
                acc[t] = __fmaf_rn(a.y, wf[1], acc[t]);
                acc[t] = __fmaf_rn(a.z, wf[2], acc[t]);
                acc[t] = __fmaf_rn(a.w, wf[3], acc[t]);
                acc[t] = __fmaf_rn(b.x, wf[4], acc[t]);
                acc[t] = __fmaf_rn(b.y, wf[5], acc[t]);
                acc[t] = __fmaf_rn(b.z, wf[6], acc[t]);
                acc[t] = __fmaf_rn(b.w, wf[7], acc[t]);
            }
        }
    };
#pragma unroll
    for (int c = 0; c < NPRE; ++c)
        if (c < nc) span(wpre[c], c);
    const uint16_t* wrow = Wr + (size_t)e * D + 8 * lane;
#pragma unroll 4
    for (int c = NPRE; c < nc; ++c) span(ld_nc_u128(wrow + 256 * c), c);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            acc[t] = __fadd_rn(acc[t], __shfl_xor_sync(0xffffffffu, acc[t], off));
    }
    if (lane == 0) {
        const float b = bias ? bias[e] : 0.0f;
#pragma unroll
        for (int t = 0; t < NT; ++t)
            if (t < nt) lout[(size_t)t * E + e] = bias ? __fadd_rn(acc[t], b) : acc[t];
    }
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp selects the top-k of one token's E logits (E <= 32 * NV) and
// writes ids and gates.  Each lane keeps its NV values and its best one; each
// of the k rounds takes the warp's best (a warp max of the value keys, then
// the lowest id among the lanes holding that key), and only the winning lane
// removes it and rescans its values.  Gates are formed in double from the
// selected fp32 logits.
template <int NV, bool SHARED = false>
__device__ void topk_warp_n(const float* __restrict__ lrow, int E, int k, int32_t* __restrict__ ids,
                            float* __restrict__ gates) {
    const int lane = threadIdx.x & 31;
    float v[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? (SHARED ? lrow[e] : __ldcg(lrow + e)) : -INFINITY;
    }
    // the lane's best: larger value, then lower id (= lower i for one lane),
    // by a pairwise tree (depth log2 NV): each pair keeps its left member
    // unless the right one is strictly larger, and the left member always
    // covers the lower indices, so equal values resolve to the lowest index
    auto rescan = [&](float& bv, int& be) {
        float tv[NV];
        int ti[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) { tv[i] = v[i]; ti[i] = i; }
#pragma unroll
        for (int st = 1; st < NV; st *= 2)
#pragma unroll
            for (int i = 0; i + st < NV; i += 2 * st)
                if (tv[i + st] > tv[i]) { tv[i] = tv[i + st]; ti[i] = ti[i + st]; }
        bv = tv[0];
        be = (lane + 32 * ti[0] < E) ? lane + 32 * ti[0] : 0x7fffffff;
    };
    float bv;
    int be;
    rescan(bv, be);
    float my_v = 0.f, l0 = 0.f;
    int my_e = 0;
    for (int r = 0; r < k; ++r) {
        const uint32_t mykey = float_key(bv);
        const uint32_t wkey = __reduce_max_sync(0xffffffffu, mykey);
        const int we = (int)__reduce_min_sync(0xffffffffu, mykey == wkey ? (uint32_t)be : 0xffffffffu);
        const float wv = __shfl_sync(0xffffffffu, bv, we & 31);
        if (r == 0) l0 = wv;
        if (lane == r) { my_v = wv; my_e = we; }
        if (be == we) {                         // this lane supplied the winner: remove it
            const int wi = (we - lane) >> 5;
#pragma unroll
            for (int i = 0; i < NV; ++i)
                if (i == wi) v[i] = -INFINITY;
            rescan(bv, be);
        }
    }
    const double ex = (lane < k) ? exp((double)my_v - (double)l0) : 0.0;
    double z = ex;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane < k) {
        ids[lane] = my_e;
        gates[lane] = (float)(ex / z);
    }
}

__device__ __forceinline__ void topk_warp(const float* __restrict__ lrow, int E, int k, int32_t* __restrict__ ids,
                                          float* __restrict__ gates) {
    if (E <= 512) topk_warp_n<16>(lrow, E, k, ids, gates);
    else topk_warp_n<32>(lrow, E, k, ids, gates);
}

// Canonical logit (+ bias) of expert e for one token (bf16 row xrow), every
// lane returning the value: the same order as canon_logits_warp.
__device__ __forceinline__ float canon_logit_one(const uint16_t* __restrict__ xrow, int D,
                                                 const uint16_t* __restrict__ Wr, const float* __restrict__ bias,
                                                 int e) {
    const int lane = threadIdx.x & 31;
    float acc = 0.0f;
    const uint16_t* wrow = Wr + (size_t)e * D + 8 * lane;
    const int nc = D >> 8;
    for (int c = 0; c < nc; ++c) {
        const uint4 w = ld_nc_u128(wrow + 256 * c);
        const uint4 xv4 = *reinterpret_cast<const uint4*>(xrow + 256 * c + 8 * lane);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        const uint32_t xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc = __fmaf_rn(bf16lo(xv[q]), bf16lo(wv[q]), acc);
            acc = __fmaf_rn(bf16hi(xv[q]), bf16hi(wv[q]), acc);
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    return bias ? __fadd_rn(acc, __ldg(bias + e)) : acc;
}

// Top-k of a row of logits held in shared memory.
__device__ __forceinline__ void topk_row_warp(const float* lrow, int E, int k, int32_t* __restrict__ ids,
                                              float* __restrict__ gates) {
    if (E <= 512) topk_warp_n<16, true>(lrow, E, k, ids, gates);
    else topk_warp_n<32, true>(lrow, E, k, ids, gates);
}

}  // namespace moe
