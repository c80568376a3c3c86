// decode.cu — expert pass for 1-4 tokens (one token plus MTP drafts):
// expert-cache slot lookup with a miss list, then a grouped dequant-GEMV that
// streams the packed codes of every selected resident expert from HBM once.
//
// The pages: experts cached in VRAM are computed on the GPU, misses elsewhere
// (wiselychen RTX 5090 report §2 "專家快取與 CPU／GPU 分工"; greenbean-ai
// "Strata 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next" §二); decode verifies MTP drafts
// in one batched pass (wiselychen report §4; greenbean-ai §三).
//
// Work: "pairs" q = t*k + r (token t's rank-r expert) plus the shared expert.
// The first pair of each distinct resident slot "owns" that expert and serves
// every token that selected it, so each expert's bytes are read once.
// Kernel 1 (gate|up) writes h = bf16(silu(Wg x) * (Wu x)); kernel 2 (down)
// writes y = Wd h as fp32 rows of expert_out.
//
// Both kernels are persistent (one CTA per SM): a producer warp streams work
// items (a block of matrix rows of one expert: codes + scales, contiguous in
// the pool) into a ring of shared-memory stages with bulk copies (TMA),
// completing on mbarriers; eight consumer warps compute from shared memory.
// Programmatic dependent launch lets kernel 2 start, resolve its work and
// prefetch its weights while kernel 1 finishes.
//
// Inner product without dequantising each weight: for a block with scale s
// and min m, sum_j (s q_j + m) x_j = s * sum_j q_j x_j + m * sum_j x_j.  Each
// code is turned into the float 2^(23-p) + q by OR-ing it, at mantissa bit p,
// into the exponent of 2^(23-p) (one logic op per code); then
// sum_j q_j x_j = sum_j x_j f_j - sum_j x_j 2^(23-p_j), the last sum being a
// per-block constant of the token computed once.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

namespace moe {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;        // + one producer warp
constexpr int kXStride = 36;                     // floats per 32-weight chunk: 32 x + 4 constants
constexpr int kMaxPairs = kDecodeMaxT * kMaxTopK + 1;
constexpr int kMaxStages = 4;
constexpr int kSmemBudget = 200 * 1024;

// ---------------------------------------------------------------- code decode
// Q2_32: code j of a 32-bit word sits at bits [2j, 2j+2).  Shifting the word by
// 21, 11, 1 or -9 places codes {0}, {1..5}, {6..10}, {11..15} at mantissa bits 13..21.
MOE_DEVINL int q2_pos(int j) { return j == 0 ? 21 : (j <= 5 ? 2 * j + 11 : (j <= 10 ? 2 * j + 1 : 2 * j - 9)); }
MOE_DEVINL float q2_code(const uint32_t* w, int i) {
    const uint32_t word = w[i >> 4];
    const int j = i & 15;
    const uint32_t src = j == 0 ? (word << 21) : (j <= 5 ? (word << 11) : (j <= 10 ? (word << 1) : (word >> 9)));
    const int p = q2_pos(j);
    return __uint_as_float((src & (3u << p)) | ((uint32_t)(150 - p) << 23));
}
// Q3 (32 codes in 3 words, code i at stream bits [3i, 3i+3)): groups of three
// codes are moved to bits 14..22, so code i sits at bit 14 + 3*(i % 3).
MOE_DEVINL int q3_pos(int i) { return 14 + 3 * (i % 3); }
MOE_DEVINL float q3_code(const uint32_t* w, int i) {
    uint32_t src;
    switch (i / 3) {
        case 0: src = w[0] << 14; break;
        case 1: src = w[0] << 5; break;
        case 2: src = w[0] >> 4; break;
        case 3: src = __funnelshift_r(w[0], w[1], 13); break;
        case 4: src = w[1] << 10; break;
        case 5: src = w[1] << 1; break;
        case 6: src = w[1] >> 8; break;
        case 7: src = __funnelshift_r(w[1], w[2], 17); break;
        case 8: src = w[2] << 6; break;
        case 9: src = w[2] >> 3; break;
        default: src = w[2] >> 12; break;
    }
    const int p = q3_pos(i);
    return __uint_as_float((src & (7u << p)) | ((uint32_t)(150 - p) << 23));
}
template <int FMT>
MOE_DEVINL float code_f(const uint32_t* w, int i) {
    if constexpr (FMT == MOE_Q2_32) return q2_code(w, i);
    else return q3_code(w, i);
}
template <int FMT>
MOE_DEVINL int code_pos(int i) {
    if constexpr (FMT == MOE_Q2_32) return q2_pos(i & 15);
    else return q3_pos(i);
}

MOE_DEVINL float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long ra, rb, rc, rd;
    asm("mov.b64 %0, {%1,%2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1,%2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1,%2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
    float2 d;
    asm("mov.b64 {%0,%1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
    return d;
}

MOE_DEVINL void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

// ---------------------------------------------------------------- format geometry
template <int FMT>
struct Geo {
    static constexpr int kCodeBytes = (FMT == MOE_Q2_32) ? 8 : 12;   // per 32-weight chunk
    static constexpr int kBlock = (FMT == MOE_Q3_S256) ? 256 : 32;
    static constexpr int kBlockCode = (FMT == MOE_Q2_32) ? 8 : (FMT == MOE_Q3_32 ? 12 : 96);
    // bytes of one matrix row with K weights, per region
    static constexpr int code_row(int K) { return K / 32 * kCodeBytes; }
    static constexpr int meta_row(int K) { return (FMT == MOE_Q3_S256) ? K / 256 * 12 : K / 32 * 4; }
    static constexpr int d_row(int K) { return (FMT == MOE_Q3_S256) ? K / 256 * 2 : 0; }
    static constexpr int row_bytes(int K) { return code_row(K) + meta_row(K) + d_row(K); }
};

struct Planes {
    const uint8_t* c;   // code plane
    const uint8_t* m;   // (s,m) plane or sub-scale plane
    const uint8_t* d;   // d plane (Q3_S256) or unused
};

template <int FMT>
MOE_DEVINL Planes planes_of(const PoolView& P, int slot, int mat) {
    const size_t blocks = (size_t)P.D * P.F / Geo<FMT>::kBlock;
    Planes pl;
    pl.c = P.codes + (size_t)slot * P.stride_c + (size_t)mat * blocks * Geo<FMT>::kBlockCode;
    const uint8_t* meta = P.scales + (size_t)slot * P.stride_s;
    if constexpr (FMT == MOE_Q3_S256) {
        pl.m = meta + (size_t)mat * blocks * 12;
        pl.d = meta + 3 * blocks * 12 + (size_t)mat * blocks * 2;
    } else {
        pl.m = meta + (size_t)mat * blocks * 4;
        pl.d = nullptr;
    }
    return pl;
}

// ---------------------------------------------------------------- work resolution
struct Owner {
    int slot;
    int ntok;
    int tok[kDecodeMaxT];
    uint32_t rmask[kDecodeMaxT];   // ranks of the token served by this expert
};

struct DecodeParams {
    PoolView P;
    const int32_t* slot_table;
    int E;
    const uint16_t* x;
    int T;
    const int32_t* ids;
    int k;
    int32_t* rowmap;       // [T][k+1]
    float* yrows;          // [T*(k+1)][D]
    int32_t* miss_list;
    int32_t* miss_count;
    uint16_t* hbuf;        // [kMaxPairs][4][F]
    uint32_t* err;
    int rf;                // gate|up: features per item
    int rd;                // down: rows per item
    int ns_gu, ns_dn;      // pipeline stages
};

struct Shared {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    Owner owners[kMaxPairs];
    int slot_of[kMaxPairs];
    int n_owners;
    int cur_owner;
};

MOE_DEVINL int lookup_slot(const DecodeParams& prm, int e) {
    int s = (e >= 0 && e < prm.E) ? __ldg(prm.slot_table + e) : -1;
    return (s < 0 || s >= prm.P.n_slots) ? -1 : s;
}

// One warp: resolve every pair's slot, the owners (first pair of each distinct
// resident slot, in pair order, then the shared expert) and, with `book`, the
// row map, miss list and miss count.
__device__ void resolve_owners(const DecodeParams& prm, Shared& sh, bool book) {
    const int lane = threadIdx.x & 31;
    const int T = prm.T, k = prm.k, n = T * k;   // n <= 64
    int e0 = -1, e1 = -1;
    for (int q = lane; q < n; q += 32) {
        const int e = __ldg(prm.ids + q);
        sh.slot_of[q] = lookup_slot(prm, e);
        if (q < 32) e0 = e; else e1 = e;
    }
    __syncwarp();
    const int s0 = lane < n ? sh.slot_of[lane] : -1;
    const int s1 = lane + 32 < n ? sh.slot_of[lane + 32] : -1;
    const uint32_t miss0 = __ballot_sync(0xffffffffu, lane < n && s0 < 0);
    const uint32_t miss1 = __ballot_sync(0xffffffffu, lane + 32 < n && s1 < 0);
    if (book) {
        const uint32_t below = (1u << lane) - 1u;
        if (lane < n) {
            const int t = lane / k, r = lane % k;
            prm.rowmap[t * (k + 1) + r] = s0 >= 0 ? t * (k + 1) + r : -1;
            if (s0 < 0) {
                const int pos = __popc(miss0 & below);
                prm.miss_list[3 * pos + 0] = t; prm.miss_list[3 * pos + 1] = r; prm.miss_list[3 * pos + 2] = e0;
            }
        }
        if (lane + 32 < n) {
            const int q = lane + 32, t = q / k, r = q % k;
            prm.rowmap[t * (k + 1) + r] = s1 >= 0 ? t * (k + 1) + r : -1;
            if (s1 < 0) {
                const int pos = __popc(miss0) + __popc(miss1 & below);
                prm.miss_list[3 * pos + 0] = t; prm.miss_list[3 * pos + 1] = r; prm.miss_list[3 * pos + 2] = e1;
            }
        }
        if (lane < T) prm.rowmap[lane * (k + 1) + k] = lane * (k + 1) + k;
        if (lane == 0) prm.miss_count[0] = __popc(miss0) + __popc(miss1);
    }
    // owners: lane handles pairs p = lane and p = lane + 32
    bool own[2] = {false, false};
    uint32_t rm[2][kDecodeMaxT];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = lane + 32 * h;
        const int sp = h == 0 ? s0 : s1;
#pragma unroll
        for (int t = 0; t < kDecodeMaxT; ++t) rm[h][t] = 0;
        if (p < n && sp >= 0) {
            bool first = true;
            for (int t = 0; t < T; ++t)
                for (int r = 0; r < k; ++r) {
                    const int q = t * k + r;
                    if (sh.slot_of[q] == sp) {
                        if (q < p) first = false;
                        rm[h][t] |= 1u << r;
                    }
                }
            own[h] = first;
        }
    }
    const uint32_t b0 = __ballot_sync(0xffffffffu, own[0]);
    const uint32_t b1 = __ballot_sync(0xffffffffu, own[1]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (own[h]) {
            const int idx = (h == 0) ? __popc(b0 & ((1u << lane) - 1u)) : __popc(b0) + __popc(b1 & ((1u << lane) - 1u));
            Owner o;
            o.slot = h == 0 ? s0 : s1;
            o.ntok = 0;
            for (int t = 0; t < T; ++t)
                if (rm[h][t]) { o.tok[o.ntok] = t; o.rmask[o.ntok] = rm[h][t]; ++o.ntok; }
            sh.owners[idx] = o;
        }
    }
    if (lane == 0) {
        const int idx = __popc(b0) + __popc(b1);
        Owner o;
        o.slot = prm.P.shared_slot;
        o.ntok = T;
        for (int t = 0; t < T; ++t) { o.tok[t] = t; o.rmask[t] = 1u << k; }
        sh.owners[idx] = o;
        sh.n_owners = idx + 1;
    }
    __syncwarp();
}

// ---------------------------------------------------------------- activations to smem
// xs[(n * nb + b) * 36 + j]: fp32 activation j of chunk b of token n; slots 32..33
// hold per-chunk constants: Q2/Q3_32: C = sum x_j 2^(23-p_j), X = sum x_j;
// Q3_S256: C'lo, C'hi = sum over the half of x_j (2^(23-p_j) + 4)  (the +4 folds
// the min -4*S of the sub-block into the constant).  Run by the consumer threads.
template <int FMT>
__device__ void stage_activations(const uint16_t* __restrict__ src, size_t tok_stride, int ntok, int K, float* xs) {
    const int nb = K / 32;
    for (int idx = threadIdx.x; idx < ntok * nb; idx += kConsumers) {
        const int n = idx / nb, b = idx - n * nb;
        const uint4* p = reinterpret_cast<const uint4*>(src + (size_t)n * tok_stride + 32 * b);
        float v[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 w = p[q];
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[8 * q + 2 * h] = bf16lo(ww[h]);
                v[8 * q + 2 * h + 1] = bf16hi(ww[h]);
            }
        }
        float* dst = xs + (size_t)idx * kXStride;
#pragma unroll
        for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        double c0 = 0.0, c1 = 0.0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const double base = (double)(1u << (23 - code_pos<FMT>(j)));
            if constexpr (FMT == MOE_Q3_S256) {
                const double c = (double)v[j] * (base + 4.0);
                if (j < 16) c0 += c; else c1 += c;
            } else {
                c0 += (double)v[j] * base;
                c1 += (double)v[j];
            }
        }
        dst[32] = (float)c0;
        dst[33] = (float)c1;
    }
}

// ---------------------------------------------------------------- one chunk, four rows
// cw[r]: the chunk's code words of row r; sa/sb: Q2/Q3_32 (s, m), Q3_S256 (S_lo, S_hi).
// xc[t]: the chunk's activations of the t-th served token.
template <int FMT, int NT>
MOE_DEVINL void chunk4(const uint32_t (&cw)[4][3], const float (&sa)[4], const float (&sb)[4],
                       const float* const (&xc)[NT], float (&res)[4][NT]) {
    constexpr int H = (FMT == MOE_Q3_S256) ? 2 : 1;
    float2 acc[4][NT][H];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int h = 0; h < H; ++h) acc[r][t][h] = make_float2(0.f, 0.f);
#pragma unroll
    for (int sc = 0; sc < 4; ++sc) {
        float xv[NT][8];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float4 a = *reinterpret_cast<const float4*>(xc[t] + 8 * sc);
            const float4 b = *reinterpret_cast<const float4*>(xc[t] + 8 * sc + 4);
            xv[t][0] = a.x; xv[t][1] = a.y; xv[t][2] = a.z; xv[t][3] = a.w;
            xv[t][4] = b.x; xv[t][5] = b.y; xv[t][6] = b.z; xv[t][7] = b.w;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const int code = 8 * sc + i;
                const float2 f = make_float2(code_f<FMT>(cw[r], code), code_f<FMT>(cw[r], code + 1));
                const int h = (H == 2 && code >= 16) ? 1 : 0;
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    acc[r][t][h] = ffma2(make_float2(xv[t][i], xv[t][i + 1]), f, acc[r][t][h]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const float c0 = xc[t][32];
        const float c1 = xc[t][33];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if constexpr (H == 2) {
                res[r][t] = __fmaf_rn(sa[r], (acc[r][t][0].x + acc[r][t][0].y) - c0, res[r][t]);
                res[r][t] = __fmaf_rn(sb[r], (acc[r][t][1].x + acc[r][t][1].y) - c1, res[r][t]);
            } else {
                res[r][t] = __fmaf_rn(sa[r], (acc[r][t][0].x + acc[r][t][0].y) - c0, __fmaf_rn(sb[r], c1, res[r][t]));
            }
        }
    }
}

// Chunk b (32 weights along K) of local row `row` of a staged item region.
// cbase/mbase/dbase: the region's code/meta/d bytes; K: row length.
template <int FMT>
MOE_DEVINL void smem_chunk(const uint8_t* cbase, const uint8_t* mbase, const uint8_t* dbase, int row, int K, int b,
                           uint32_t (&w)[3], float& sa, float& sb) {
    if constexpr (FMT == MOE_Q2_32) {
        const uint2 c = *reinterpret_cast<const uint2*>(cbase + (size_t)row * Geo<FMT>::code_row(K) + b * 8);
        w[0] = c.x; w[1] = c.y; w[2] = 0;
        const uint32_t sm = *reinterpret_cast<const uint32_t*>(mbase + (size_t)row * Geo<FMT>::meta_row(K) + b * 4);
        sa = f16_bits_to_f32(sm & 0xffffu);
        sb = f16_bits_to_f32(sm >> 16);
    } else if constexpr (FMT == MOE_Q3_32) {
        const uint32_t* p = reinterpret_cast<const uint32_t*>(cbase + (size_t)row * Geo<FMT>::code_row(K) + b * 12);
        w[0] = p[0]; w[1] = p[1]; w[2] = p[2];
        const uint32_t sm = *reinterpret_cast<const uint32_t*>(mbase + (size_t)row * Geo<FMT>::meta_row(K) + b * 4);
        sa = f16_bits_to_f32(sm & 0xffffu);
        sb = f16_bits_to_f32(sm >> 16);
    } else {
        const int sbk = b >> 3, j = b & 7;
        const uint32_t* p = reinterpret_cast<const uint32_t*>(cbase + (size_t)row * Geo<FMT>::code_row(K) + b * 12);
        w[0] = p[0]; w[1] = p[1]; w[2] = p[2];
        const uint32_t* scp = reinterpret_cast<const uint32_t*>(mbase + (size_t)row * Geo<FMT>::meta_row(K) + sbk * 12);
        const int bit = 12 * j, wi = bit >> 5, sh = bit & 31;
        const uint32_t lo = scp[wi];
        const uint32_t hi = wi < 2 ? scp[wi + 1] : 0u;
        const uint32_t bits = __funnelshift_r(lo, hi, sh);
        const float d = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(dbase + (size_t)row * Geo<FMT>::d_row(K) + sbk * 2));
        sa = d * (float)((int)(bits & 63u) - 32);          // exact
        sb = d * (float)((int)((bits >> 6) & 63u) - 32);
    }
}

MOE_DEVINL float silu_f(float g) { return g / (1.0f + expf(-g)); }

// Issue the bulk copies of `nrows` rows starting at `row0` of matrix planes pl
// (rows of K weights) into dst (codes | meta | d), completing on bar.
template <int FMT>
MOE_DEVINL void issue_rows(const Planes& pl, int row0, int nrows, int K, uint8_t* dst, uint64_t* bar) {
    const uint32_t cr = Geo<FMT>::code_row(K), mr = Geo<FMT>::meta_row(K), dr = Geo<FMT>::d_row(K);
    bulk_g2s(dst, pl.c + (size_t)row0 * cr, cr * nrows, bar);
    bulk_g2s(dst + cr * nrows, pl.m + (size_t)row0 * mr, mr * nrows, bar);
    if constexpr (FMT == MOE_Q3_S256) bulk_g2s(dst + (cr + mr) * nrows, pl.d + (size_t)row0 * dr, dr * nrows, bar);
}

// ---------------------------------------------------------------- gate | up
// Item = (owner u, features [f0, f0 + rf)); staged as gate rows then up rows.
template <int FMT, int NT>
__device__ void gateup_item(const DecodeParams& prm, const Owner& o, int u, int f0, const uint8_t* stage,
                            const float* xs) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F, rf = prm.rf;
    const int nb = D / 32;
    const int lpr = min(32, nb & -nb);
    const int G = 32 / lpr, group = lane / lpr, gl = lane % lpr;
    const uint32_t cr = Geo<FMT>::code_row(D), mr = Geo<FMT>::meta_row(D);
    const uint32_t half = (uint32_t)Geo<FMT>::row_bytes(D) * rf;   // gate rows then up rows
    const uint8_t* gc = stage;
    const uint8_t* gm = stage + cr * rf;
    const uint8_t* gd = stage + (cr + mr) * rf;
    const uint8_t* uc = stage + half;
    const uint8_t* um = uc + cr * rf;
    const uint8_t* ud = uc + (cr + mr) * rf;
    for (int q = warp * G + group; q < rf / 2; q += kConsumerWarps * G) {
        const int fl = 2 * q;   // local feature
        float res[4][NT];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t) res[r][t] = 0.f;
        for (int b = gl; b < nb; b += lpr) {
            uint32_t cw[4][3];
            float sa[4], sb[4];
            smem_chunk<FMT>(gc, gm, gd, fl, D, b, cw[0], sa[0], sb[0]);
            smem_chunk<FMT>(gc, gm, gd, fl + 1, D, b, cw[1], sa[1], sb[1]);
            smem_chunk<FMT>(uc, um, ud, fl, D, b, cw[2], sa[2], sb[2]);
            smem_chunk<FMT>(uc, um, ud, fl + 1, D, b, cw[3], sa[3], sb[3]);
            const float* xc[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) xc[t] = xs + ((size_t)o.tok[t] * nb + b) * kXStride;
            chunk4<FMT, NT>(cw, sa, sb, xc, res);
        }
        for (int off = lpr >> 1; off >= 1; off >>= 1)
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int t = 0; t < NT; ++t) res[r][t] += __shfl_xor_sync(0xffffffffu, res[r][t], off);
        if (gl == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint16_t h0 = f32_to_bf16_rne(silu_f(res[0][t]) * res[2][t]);
                const uint16_t h1 = f32_to_bf16_rne(silu_f(res[1][t]) * res[3][t]);
                *reinterpret_cast<uint32_t*>(prm.hbuf + ((size_t)u * kDecodeMaxT + t) * F + f0 + fl) =
                    (uint32_t)h0 | ((uint32_t)h1 << 16);
            }
        }
    }
}

template <int FMT, int NTMAX>
__global__ void __launch_bounds__(kThreads, 1) decode_gateup_kernel(DecodeParams prm) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ Shared sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F, rf = prm.rf, NS = prm.ns_gu;
    const int nb = D / 32;
    const size_t xs_bytes = ((size_t)prm.T * nb * kXStride * 4 + 127) / 128 * 128;
    float* xs = reinterpret_cast<float*>(smem);
    uint8_t* stages = smem + xs_bytes;
    const uint32_t item_bytes = 2u * Geo<FMT>::row_bytes(D) * rf;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], kConsumerWarps); }
        fence_mbar_init();
    }
    pdl_wait();                      // ids come from the router
    if (warp == 0) resolve_owners(prm, sh, blockIdx.x == 0);
    __syncthreads();
    pdl_launch_dependents();         // the down kernel may start its prologue
    const int nfb = F / rf;
    const int n_items = sh.n_owners * nfb;
    if (warp == kConsumerWarps) {    // producer: round-robin items
        if (lane == 0) {
            int j = 0;
            for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++j) {
                const int s = j % NS;
                if (j >= NS && !mbar_wait(&sh.empty[s], ((j / NS) - 1) & 1, prm.err)) break;
                const int u = i / nfb, f0 = (i % nfb) * rf;
                const int slot = sh.owners[u].slot;
                uint8_t* dst = stages + (size_t)s * item_bytes;
                mbar_arrive_expect_tx(&sh.full[s], item_bytes);
                issue_rows<FMT>(planes_of<FMT>(prm.P, slot, 0), f0, rf, D, dst, &sh.full[s]);
                issue_rows<FMT>(planes_of<FMT>(prm.P, slot, 1), f0, rf, D, dst + item_bytes / 2, &sh.full[s]);
            }
        }
        return;
    }
    stage_activations<FMT>(prm.x, D, prm.T, D, xs);
    consumer_sync();
    int j = 0;
    for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++j) {
        const int s = j % NS;
        if (!mbar_wait(&sh.full[s], (j / NS) & 1, prm.err)) return;
        const int u = i / nfb, f0 = (i % nfb) * rf;
        const Owner& o = sh.owners[u];
        const uint8_t* st = stages + (size_t)s * item_bytes;
        if constexpr (NTMAX == 1) {
            gateup_item<FMT, 1>(prm, o, u, f0, st, xs);
        } else {
            switch (o.ntok) {
                case 1: gateup_item<FMT, 1>(prm, o, u, f0, st, xs); break;
                case 2: gateup_item<FMT, 2>(prm, o, u, f0, st, xs); break;
                case 3: gateup_item<FMT, 3>(prm, o, u, f0, st, xs); break;
                default: gateup_item<FMT, 4>(prm, o, u, f0, st, xs); break;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
    }
}

// ---------------------------------------------------------------- down
// Item = (owner u, rows [d0, d0 + rd)) of Wd.  Items are split in contiguous
// ranges per CTA so that consecutive items mostly share the owner (h is
// re-staged only when the owner changes).
template <int FMT, int NT>
__device__ void down_item(const DecodeParams& prm, const Owner& o, int d0, const uint8_t* stage, const float* hs) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F, k = prm.k, rd = prm.rd;
    const int nb = F / 32;
    const int lpr = min(32, nb & -nb);
    const int G = 32 / lpr, group = lane / lpr, gl = lane % lpr;
    const uint32_t cr = Geo<FMT>::code_row(F), mr = Geo<FMT>::meta_row(F);
    const uint8_t* dc = stage;
    const uint8_t* dm = stage + cr * rd;
    const uint8_t* dd = stage + (cr + mr) * rd;
    for (int q = warp * G + group; q < rd / 4; q += kConsumerWarps * G) {
        const int rl = 4 * q;
        float res[4][NT];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t) res[r][t] = 0.f;
        for (int b = gl; b < nb; b += lpr) {
            uint32_t cw[4][3];
            float sa[4], sb[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) smem_chunk<FMT>(dc, dm, dd, rl + r, F, b, cw[r], sa[r], sb[r]);
            const float* xc[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) xc[t] = hs + ((size_t)t * nb + b) * kXStride;
            chunk4<FMT, NT>(cw, sa, sb, xc, res);
        }
        for (int off = lpr >> 1; off >= 1; off >>= 1)
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int t = 0; t < NT; ++t) res[r][t] += __shfl_xor_sync(0xffffffffu, res[r][t], off);
        if (gl == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float4 v = make_float4(res[0][t], res[1][t], res[2][t], res[3][t]);
                uint32_t m = o.rmask[t];
                while (m) {
                    const int r = __ffs(m) - 1;
                    m &= m - 1;
                    *reinterpret_cast<float4*>(prm.yrows + ((size_t)o.tok[t] * (k + 1) + r) * D + d0 + rl) = v;
                }
            }
        }
    }
}

template <int FMT, int NTMAX>
__global__ void __launch_bounds__(kThreads, 1) decode_down_kernel(DecodeParams prm) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ Shared sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F, rd = prm.rd, NS = prm.ns_dn;
    const int nb = F / 32;
    const size_t hs_bytes = ((size_t)kDecodeMaxT * nb * kXStride * 4 + 127) / 128 * 128;
    float* hs = reinterpret_cast<float*>(smem);
    uint8_t* stages = smem + hs_bytes;
    const uint32_t item_bytes = (uint32_t)Geo<FMT>::row_bytes(F) * rd;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], kConsumerWarps); }
        fence_mbar_init();
        sh.cur_owner = -1;
    }
    // ids and the slot table were complete before the gate|up kernel passed its
    // own dependency wait, which precedes the launch of this grid: the owners can
    // be resolved and the down weights prefetched before waiting for h.
    if (warp == 0) resolve_owners(prm, sh, false);
    __syncthreads();
    const int nrb = D / rd;
    const int n_items = sh.n_owners * nrb;
    const int per = (n_items + gridDim.x - 1) / gridDim.x;
    const int i0 = blockIdx.x * per, i1 = min(n_items, i0 + per);
    if (warp == kConsumerWarps) {
        if (lane == 0) {
            for (int i = i0, j = 0; i < i1; ++i, ++j) {
                const int s = j % NS;
                if (j >= NS && !mbar_wait(&sh.empty[s], ((j / NS) - 1) & 1, prm.err)) break;
                const int u = i / nrb, d0 = (i % nrb) * rd;
                mbar_arrive_expect_tx(&sh.full[s], item_bytes);
                issue_rows<FMT>(planes_of<FMT>(prm.P, sh.owners[u].slot, 2), d0, rd, F, stages + (size_t)s * item_bytes,
                                &sh.full[s]);
            }
        }
        return;
    }
    pdl_wait();                      // h comes from the gate|up kernel
    pdl_launch_dependents();
    int cur = -1;
    for (int i = i0, j = 0; i < i1; ++i, ++j) {
        const int s = j % NS;
        const int u = i / nrb, d0 = (i % nrb) * rd;
        const Owner& o = sh.owners[u];
        if (u != cur) {
            consumer_sync();
            stage_activations<FMT>(prm.hbuf + (size_t)u * kDecodeMaxT * F, F, o.ntok, F, hs);
            consumer_sync();
            cur = u;
        }
        if (!mbar_wait(&sh.full[s], (j / NS) & 1, prm.err)) return;
        const uint8_t* st = stages + (size_t)s * item_bytes;
        if constexpr (NTMAX == 1) {
            down_item<FMT, 1>(prm, o, d0, st, hs);
        } else {
            switch (o.ntok) {
                case 1: down_item<FMT, 1>(prm, o, d0, st, hs); break;
                case 2: down_item<FMT, 2>(prm, o, d0, st, hs); break;
                case 3: down_item<FMT, 3>(prm, o, d0, st, hs); break;
                default: down_item<FMT, 4>(prm, o, d0, st, hs); break;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
    }
}

int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int FMT, int NTMAX>
moe_status launch_fmt(DecodeParams prm, cudaStream_t s) {
    const int T = prm.T, D = prm.P.D, F = prm.P.F;
    // gate|up: features per item and stages so that x + stages fit the budget
    const size_t xs_bytes = ((size_t)T * (D / 32) * kXStride * 4 + 127) / 128 * 128;
    int rf = 16;
    while (rf > 2 && xs_bytes + 2 * 2 * (size_t)Geo<FMT>::row_bytes(D) * rf > 150 * 1024) rf /= 2;
    prm.rf = rf;
    prm.ns_gu = 2;
    const size_t smem1 = xs_bytes + (size_t)prm.ns_gu * 2 * Geo<FMT>::row_bytes(D) * rf;
    // down: rows per item and stages within ~100 KB (co-resident with gate|up)
    const size_t hs_bytes = ((size_t)kDecodeMaxT * (F / 32) * kXStride * 4 + 127) / 128 * 128;
    int rd = 128;
    while (rd > 16 && hs_bytes + 3 * (size_t)Geo<FMT>::row_bytes(F) * rd > 100 * 1024) rd /= 2;
    prm.rd = rd;
    prm.ns_dn = 3;
    const size_t smem2 = hs_bytes + (size_t)prm.ns_dn * Geo<FMT>::row_bytes(F) * rd;
    if (smem1 > kSmemBudget || smem2 > kSmemBudget || F % rf || D % rd) return MOE_ERR_UNSUPPORTED;
    static bool attr_done = false;
    if (!attr_done) {
        cudaFuncSetAttribute(decode_gateup_kernel<FMT, NTMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
        cudaFuncSetAttribute(decode_down_kernel<FMT, NTMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
        attr_done = true;
    }
    const int grid = num_sms();
    cudaError_t e = launch_pdl(decode_gateup_kernel<FMT, NTMAX>, dim3(grid), dim3(kThreads), smem1, s, prm);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_pdl(decode_down_kernel<FMT, NTMAX>, dim3(grid), dim3(kThreads), smem2, s, prm);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

size_t decode_workspace_bytes(int T, int D, int F, int k) {
    (void)D; (void)T; (void)k;
    return 256 + (size_t)kMaxPairs * kDecodeMaxT * F * sizeof(uint16_t);
}

moe_status launch_decode_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x, int T,
                                 const int32_t* ids, int k, void* expert_out, int32_t* miss_list,
                                 int32_t* miss_count, void* ws, cudaStream_t s) {
    DecodeParams prm;
    prm.P = P;
    prm.slot_table = slot_table;
    prm.E = E;
    prm.x = x;
    prm.T = T;
    prm.ids = ids;
    prm.k = k;
    prm.rowmap = reinterpret_cast<int32_t*>(expert_out);
    prm.yrows = reinterpret_cast<float*>(reinterpret_cast<char*>(expert_out) + rowmap_bytes(T, k));
    prm.miss_list = miss_list;
    prm.miss_count = miss_count;
    prm.err = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 4);
    prm.hbuf = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(ws) + 256);
    const bool one = (T == 1);
    switch (P.fmt) {
        case MOE_Q2_32: return one ? launch_fmt<MOE_Q2_32, 1>(prm, s) : launch_fmt<MOE_Q2_32, 4>(prm, s);
        case MOE_Q3_32: return one ? launch_fmt<MOE_Q3_32, 1>(prm, s) : launch_fmt<MOE_Q3_32, 4>(prm, s);
        default: return one ? launch_fmt<MOE_Q3_S256, 1>(prm, s) : launch_fmt<MOE_Q3_S256, 4>(prm, s);
    }
}

}  // namespace moe
