// route_warp.cuh — warp-level router pieces shared by the decode and prefill
// routers: logits in the canonical fp32 order and the top-k selection.
#pragma once

#include "common.cuh"

namespace moe {

// Position of element d of a token row in the fp32 staging layout of the
// decode router: within each 256-element span, elements j = 0..3 of lane L's
// eight sit at 4L + j and elements j = 4..7 at 128 + 4L + (j - 4), so each of a
// lane's two 16-byte reads is one contiguous 512-byte sweep of the warp.
__device__ __forceinline__ int canon_stage_pos(int d) {
    const int c = d >> 8, L = (d >> 3) & 31, j = d & 7;
    return (c << 8) + ((j >> 2) << 7) + (L << 2) + (j & 3);
}

// Stage T bf16 token rows [T][D] into xsf as fp32 in the canon_stage_pos
// layout, threads tid = 0..nthreads-1 of the caller; every load of a batch is
// in flight before the first store.
__device__ __forceinline__ void stage_x_canon(const uint16_t* __restrict__ x, int T, int D, float* xsf, int tid,
                                              int nthreads) {
    constexpr int kBatch = 16;
    const int n16 = T * D / 8;
    for (int i0 = 0; i0 < n16; i0 += kBatch * nthreads) {
        uint4 v[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int i = i0 + q * nthreads + tid;
            v[q] = i < n16 ? __ldg(reinterpret_cast<const uint4*>(x) + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int i = i0 + q * nthreads + tid;
            if (i < n16) {
                const int t = (8 * i) / D, d = 8 * i - t * D;
                float* dst = xsf + (size_t)t * D + canon_stage_pos(d);
                *reinterpret_cast<float4*>(dst) = make_float4(bf16lo(v[q].x), bf16hi(v[q].x), bf16lo(v[q].y), bf16hi(v[q].y));
                *reinterpret_cast<float4*>(dst + 128) = make_float4(bf16lo(v[q].z), bf16hi(v[q].z), bf16lo(v[q].w), bf16hi(v[q].w));
            }
        }
    }
}

// Canonical logits of expert e for NT tokens: lane L accumulates elements
// 256c + 8L + j (c ascending), then the xor butterfly, then + bias.  The token
// rows are staged in shared memory as fp32 (exact copies of the bf16 values)
// in the canon_stage_pos layout, the expert's Wr row is in shared memory too,
// and its bias (if any) in a register.
template <int NT>
__device__ __forceinline__ void canon_logits_warp_staged(const float* __restrict__ xs /* [NT][D] */, int nt, int D,
                                                         const uint16_t* __restrict__ wrow_s, bool has_bias,
                                                         float bias_e, int E, int e,
                                                         float* __restrict__ lout /* + t*E */) {
    const int lane = threadIdx.x & 31;
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
    const int nc = D >> 8;
#pragma unroll 2
    for (int c = 0; c < nc; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(wrow_s + 256 * c + 8 * lane);
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
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            acc[t] = __fadd_rn(acc[t], __shfl_xor_sync(0xffffffffu, acc[t], off));
    }
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < NT; ++t)
            if (t < nt) lout[(size_t)t * E + e] = has_bias ? __fadd_rn(acc[t], bias_e) : acc[t];
    }
}

// The same logits (same order, same arithmetic) with the token rows staged as
// bf16 [nt][D] in natural order in shared memory and the expert's Wr row read
// from shared memory (W_SHARED) or global memory (eight 16-byte loads of a
// lane in flight at a time).
template <int NT, bool W_SHARED>
__device__ __forceinline__ void canon_logits_warp_xbf16(const uint16_t* __restrict__ xs /* [NT][D] */, int nt, int D,
                                                        const uint16_t* __restrict__ wrow, bool has_bias,
                                                        float bias_e, int E, int e,
                                                        float* __restrict__ lout /* + t*E */) {
    const int lane = threadIdx.x & 31;
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
    const int nc = D >> 8;
    for (int c0 = 0; c0 < nc; c0 += 8) {
        uint4 wl[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            wl[i] = c0 + i >= nc ? make_uint4(0, 0, 0, 0)
                    : W_SHARED ? *reinterpret_cast<const uint4*>(wrow + 256 * (c0 + i) + 8 * lane)
                               : ld_nc_u128(wrow + 256 * (c0 + i) + 8 * lane);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (c0 + i < nc) {
                const int c = c0 + i;
                const uint32_t wv[4] = {wl[i].x, wl[i].y, wl[i].z, wl[i].w};
                float wf[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) { wf[2 * q] = bf16lo(wv[q]); wf[2 * q + 1] = bf16hi(wv[q]); }
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (t < nt) {
                        const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)t * D + 256 * c + 8 * lane);
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            acc[t] = __fmaf_rn(bf16lo(xw[q]), wf[2 * q], acc[t]);
                            acc[t] = __fmaf_rn(bf16hi(xw[q]), wf[2 * q + 1], acc[t]);
                        }
                    }
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
#pragma unroll
        for (int t = 0; t < NT; ++t)
            if (t < nt) lout[(size_t)t * E + e] = has_bias ? __fadd_rn(acc[t], bias_e) : acc[t];
    }
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Selection key of (logit, id): larger logit first, equal logits lower id
// first, as one unsigned 64-bit order (-0.0 is taken as +0.0 before keying).
__device__ __forceinline__ uint64_t sel_key(float v, int id) {
    return ((uint64_t)float_key(v) << 32) | (uint64_t)(~(uint32_t)id);
}
__device__ __forceinline__ float key_value(uint64_t key) {
    const uint32_t h = (uint32_t)(key >> 32);
    return __uint_as_float((h & 0x80000000u) ? (h & 0x7fffffffu) : ~h);
}
__device__ __forceinline__ int key_id(uint64_t key) { return (int)(~(uint32_t)key); }

// One warp selects the top-k of one token's E logits (E <= 32 * NV) and
// writes ids and gates.  Each lane holds NV logits (ids lane + 32 i).
// Fast path: the k-th largest of the 32 lane maxima is a threshold that at
// least k logits reach, so the top-k lie among the logits at or above it;
// when those candidates fit one per lane, each candidate's rank among them
// is counted directly.  Otherwise k tournament rounds (warp max of the
// lanes' best keys; the winning lane drops it and rescans).  Gates are formed
// in double from the selected fp32 logits.
template <int NV, bool SHARED = false>
__device__ void topk_warp_n(const float* __restrict__ lrow, int E, int k, int32_t* __restrict__ ids,
                            float* __restrict__ gates) {
    __shared__ uint64_t s_keys[8][32];   // per warp: lane maxima, then the candidates
    __shared__ uint64_t s_sel[8][32];    // per warp: the selected keys by rank
    __shared__ int s_n[8];               // per warp: candidates placed so far
    const int lane = threadIdx.x & 31, w = (threadIdx.x >> 5) & 7;
    uint64_t key[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        const float raw = (e < E) ? (SHARED ? lrow[e] : __ldcg(lrow + e)) : -INFINITY;
        key[i] = sel_key(__fadd_rn(raw, 0.0f), e < E ? e : 0x7fffffff);
    }
    // the lane's best key, by a pairwise tree
    auto lane_best = [&]() {
        uint64_t t[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) t[i] = key[i];
#pragma unroll
        for (int st = 1; st < NV; st *= 2)
#pragma unroll
            for (int i = 0; i + st < NV; i += 2 * st) t[i] = t[i + st] > t[i] ? t[i + st] : t[i];
        return t[0];
    };
    uint64_t best = lane_best();
    s_keys[w][lane] = best;
    if (lane == 0) s_n[w] = 0;
    __syncwarp();
    int above = 0;                           // lane maxima larger than this lane's
#pragma unroll
    for (int i = 0; i < 32; ++i) above += s_keys[w][i] > best;
    const uint32_t at_k = __ballot_sync(0xffffffffu, above == k - 1);   // keys are distinct: one lane
    const uint64_t tau = __shfl_sync(0xffffffffu, best, __ffs(at_k) - 1);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) cnt += key[i] >= tau;
    const int total = (int)__reduce_add_sync(0xffffffffu, (uint32_t)cnt);
    uint64_t my = 0;
    if (total <= 32) {
        // the candidates in any order (each one's rank among them is counted)
        __syncwarp();
        int pos = cnt ? atomicAdd(&s_n[w], cnt) : 0;
#pragma unroll
        for (int i = 0; i < NV; ++i)
            if (key[i] >= tau) s_keys[w][pos++] = key[i];
        __syncwarp();
        if (lane < total) {
            const uint64_t c = s_keys[w][lane];
            int rank = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) rank += (i < total && s_keys[w][i] > c);
            if (rank < k) s_sel[w][rank] = c;
        }
        __syncwarp();
        if (lane < k) my = s_sel[w][lane];
        __syncwarp();
    } else {
        for (int r = 0; r < k; ++r) {
            const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32));
            const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
            const uint64_t wk = ((uint64_t)hi << 32) | lo;
            if (lane == r) my = wk;
            if (best == wk) {                // this lane supplied the winner: drop it
#pragma unroll
                for (int i = 0; i < NV; ++i)
                    if (key[i] == wk) key[i] = 0;
                best = lane_best();
            }
        }
    }
    const float my_v = key_value(my);
    const float l0 = __shfl_sync(0xffffffffu, my_v, 0);
    const double ex = (lane < k) ? exp((double)my_v - (double)l0) : 0.0;
    double z = ex;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane < k) {
        ids[lane] = key_id(my);
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
