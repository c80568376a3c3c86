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
// Phase 1 (gate|up) writes h = bf16(silu(Wg x) * (Wu x)); phase 2 (down)
// writes y = Wd h as fp32 rows of expert_out.
//
// One persistent kernel (one CTA per SM) runs both phases: a producer warp
// streams work items (a block of matrix rows of one expert: codes + scales,
// contiguous in the pool) into a ring of shared-memory stages with bulk copies
// (TMA), completing on mbarriers; sixteen consumer warps compute from shared
// memory.  Programmatic dependent launch overlaps its prologue with the router.
//
// Inner product without dequantising each weight: for a block with scale s
// and min m, sum_j (s q_j + m) x_j = s * sum_j q_j x_j + m * sum_j x_j.  Each
// code, left at mantissa bit p_j of its word, is OR-ed into 1.0f (one logic op
// per code, one shared constant): f_j = 1 + q_j 2^(p_j - 23), exactly.  The
// staged activations are pre-scaled, x'_j = x_j 2^(23 - p_j) (exact), so that
// sum_j x'_j f_j = sum_j x'_j + sum_j q_j x_j, the first sum being a per-block
// constant of the token computed once.
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "once.cuh"
#include "sync.cuh"

namespace moe {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kTeams = 2;                        // consumer teams, alternating items
constexpr int kTeamWarps = kConsumerWarps / kTeams;
constexpr int kProducerWarp = kConsumerWarps;    // bulk copies into the stage ring
constexpr int kPublisherWarp = kConsumerWarps + 1; // releases finished gate|up items to other CTAs
constexpr int kThreads = kConsumers + 64;
constexpr int kXStride = 36;                     // floats per 32-weight chunk: 32 x + 4 constants
constexpr int kMaxPairs = kDecodeMaxT * kMaxTopK + 1;
constexpr int kMaxStages = 8;
constexpr int kSmemBudget = 220 * 1024;

// ---------------------------------------------------------------- code decode
// Q2_32: code j of a 32-bit word sits at bits [2j, 2j+2).  Shifting the word by
// 21, 11, 1 or -9 places codes {0}, {1..5}, {6..10}, {11..15} at mantissa bits 13..21.
MOE_DEVINL int q2_pos(int j) { return j == 0 ? 21 : (j <= 5 ? 2 * j + 11 : (j <= 10 ? 2 * j + 1 : 2 * j - 9)); }
// Q3 (32 codes in 3 words, code i at stream bits [3i, 3i+3)): groups of three
// codes are moved to bits 14..22, so code i sits at bit 14 + 3*(i % 3).
MOE_DEVINL int q3_pos(int i) { return 14 + 3 * (i % 3); }
// Compile-time loop: f(std::integral_constant<int, I>) for I in [B, E).
template <int B, int E, typename Fn>
MOE_DEVINL void static_for(Fn&& fn) {
    if constexpr (B < E) {
        fn(std::integral_constant<int, B>{});
        static_for<B + 1, E>(fn);
    }
}

// 1.0f as a register operand the compiler cannot fold: `(src & mask) | one`
// must stay one 3-input logic op (lop3 encodes a single immediate, so two
// immediates would cost two logic ops per code on the half-rate ALU pipe).
MOE_DEVINL uint32_t opaque_one() {
    uint32_t v;
    asm volatile("mov.b32 %0, 0x3f800000;" : "=r"(v));
    return v;
}
template <uint32_t MASK>
MOE_DEVINL float and_or(uint32_t src, uint32_t one) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(src), "n"(MASK), "r"(one));   // (a & b) | c
    return __uint_as_float(r);
}

// Code I of a chunk as 1 + q 2^(p-23), with I a compile-time constant so that
// the shift and mask are immediates.
template <int FMT, int I>
MOE_DEVINL float code_c(const uint32_t* w, uint32_t one) {
    if constexpr (FMT == MOE_Q2_32) {
        constexpr int j = I & 15;
        constexpr int sh = j == 0 ? 21 : (j <= 5 ? 11 : (j <= 10 ? 1 : -9));
        constexpr int p = j == 0 ? 21 : (j <= 5 ? 2 * j + 11 : (j <= 10 ? 2 * j + 1 : 2 * j - 9));
        const uint32_t word = w[I >> 4];
        const uint32_t src = sh >= 0 ? (word << (sh >= 0 ? sh : 0)) : (word >> (sh < 0 ? -sh : 0));
        return and_or<(3u << p)>(src, one);
    } else {
        constexpr int g = I / 3;
        constexpr int p = 14 + 3 * (I % 3);
        uint32_t src;
        if constexpr (g == 0) src = w[0] << 14;
        else if constexpr (g == 1) src = w[0] << 5;
        else if constexpr (g == 2) src = w[0] >> 4;
        else if constexpr (g == 3) src = __funnelshift_r(w[0], w[1], 13);
        else if constexpr (g == 4) src = w[1] << 10;
        else if constexpr (g == 5) src = w[1] << 1;
        else if constexpr (g == 6) src = w[1] >> 8;
        else if constexpr (g == 7) src = __funnelshift_r(w[1], w[2], 17);
        else if constexpr (g == 8) src = w[2] << 6;
        else if constexpr (g == 9) src = w[2] >> 3;
        else src = w[2] >> 12;
        return and_or<(7u << p)>(src, one);
    }
}
template <int FMT>
MOE_DEVINL int code_pos(int i) {
    if constexpr (FMT == MOE_Q2_32) return q2_pos(i & 15);
    else return q3_pos(i);
}

MOE_DEVINL float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

MOE_DEVINL void team_sync(int team) { asm volatile("bar.sync %0, %1;" ::"r"(2 + team), "n"(kTeamWarps * 32) : "memory"); }
// A team barrier that also returns whether v held on every thread of the team.
MOE_DEVINL bool team_all(int team, bool v) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)v), "r"(2 + team), "n"(kTeamWarps * 32) : "memory");
    return r != 0;
}

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
    uint32_t* done;        // [kMaxPairs + 1]: per-owner gate|up completion counters + CTA ticket
    int rf;                // gate|up: features per item
    int rd;                // down: rows per item
    int ns_gu, ns_dn;      // pipeline stages
};

constexpr int kMaxE = 1024;

struct Shared {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    Owner owners[kMaxPairs];
    int slot_of[kMaxPairs];
    int table[kMaxE];          // the slot table, staged before the dependency wait
    int n_owners;
    int abort[kTeams];         // set by a consumer team that stopped on an error
    int d_range[2];            // this CTA's down items [d_range[0], d_range[1])
    uint64_t range_bar;        // completes once d_range is written
    uint32_t team_items[kTeams];   // gate|up items finished by each team (release.cta by its leader)
};

// The slot table is an input of the layer, not produced by the router: stage it
// while the router may still run.
__device__ void stage_table(const DecodeParams& prm, Shared& sh) {
    for (int e = threadIdx.x; e < prm.E; e += blockDim.x) {
        const int s = __ldg(prm.slot_table + e);
        sh.table[e] = (s < 0 || s >= prm.P.n_slots) ? -1 : s;
    }
}

// Work items.  Owner 0 (the shared expert, which serves every token and so
// costs about twice as much per row) is cut into half-size items, so that
// equal item counts are roughly equal work:
//   gate|up: 2*nfb shared items of rf/2 features, then nfb items of rf per owner
//   down   : 2*nrb shared items of rd/2 rows,     then nrb items of rd per owner
struct ItemPos { int u, row0, nrows; };
MOE_DEVINL ItemPos item_pos(int i, int per_owner, int rows) {
    ItemPos p;
    if (i < 2 * per_owner) { p.u = 0; p.nrows = rows / 2; p.row0 = i * p.nrows; }
    else { const int r = i - 2 * per_owner; p.u = 1 + r / per_owner; p.nrows = rows; p.row0 = (r % per_owner) * rows; }
    return p;
}
MOE_DEVINL int items_of(int n_owners, int per_owner) { return 2 * per_owner + (n_owners - 1) * per_owner; }

MOE_DEVINL int lookup_slot(const DecodeParams& prm, const Shared& sh, int e) {
    return (e >= 0 && e < prm.E) ? sh.table[e] : -1;
}

// One warp: resolve every pair's slot and the owners — owner 0 is the shared
// expert, then the first pair of each distinct resident slot in pair order —
// and, with `book`, the row map, miss list and miss count.
__device__ void resolve_owners(const DecodeParams& prm, Shared& sh, bool book) {
    const int lane = threadIdx.x & 31;
    const int T = prm.T, k = prm.k, n = T * k;   // n <= 64
    const int e0 = lane < n ? __ldg(prm.ids + lane) : -1;
    const int e1 = lane + 32 < n ? __ldg(prm.ids + lane + 32) : -1;
    const int s0 = lane < n ? lookup_slot(prm, sh, e0) : -1;
    const int s1 = lane + 32 < n ? lookup_slot(prm, sh, e1) : -1;
    if (lane < n) sh.slot_of[lane] = s0;
    if (lane + 32 < n) sh.slot_of[lane + 32] = s1;
    const uint32_t miss0 = __ballot_sync(0xffffffffu, lane < n && s0 < 0);
    const uint32_t miss1 = __ballot_sync(0xffffffffu, lane + 32 < n && s1 < 0);
    const uint32_t below = (1u << lane) - 1u;
    if (book) {
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
    __syncwarp();
    // lane handles pairs p = lane (h = 0) and p = lane + 32 (h = 1)
    uint32_t rm0[kDecodeMaxT] = {0, 0, 0, 0}, rm1[kDecodeMaxT] = {0, 0, 0, 0};
    bool own0 = lane < n && s0 >= 0, own1 = lane + 32 < n && s1 >= 0;
    uint64_t eq0 = 0, eq1 = 0;                 // pairs q with the same slot
#pragma unroll 8
    for (int q = 0; q < n; ++q) {
        const int sq = sh.slot_of[q];
        if (sq == s0) eq0 |= 1ull << q;
        if (sq == s1) eq1 |= 1ull << q;
    }
    if (own0 && (eq0 & ((1ull << lane) - 1ull))) own0 = false;
    if (own1 && (eq1 & ((1ull << (lane + 32)) - 1ull))) own1 = false;
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) {
        if (t < T) {
            rm0[t] = (uint32_t)(eq0 >> (t * k)) & ((1u << k) - 1u);
            rm1[t] = (uint32_t)(eq1 >> (t * k)) & ((1u << k) - 1u);
        }
    }
    const uint32_t b0 = __ballot_sync(0xffffffffu, own0);
    const uint32_t b1 = __ballot_sync(0xffffffffu, own1);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const bool own = h == 0 ? own0 : own1;
        if (own) {
            const int idx = h == 0 ? 1 + __popc(b0 & below) : 1 + __popc(b0) + __popc(b1 & below);
            Owner& o = sh.owners[idx];
            int nt = 0;
#pragma unroll
            for (int t = 0; t < kDecodeMaxT; ++t) {
                const uint32_t m = h == 0 ? rm0[t] : rm1[t];
                if (t < T && m) { o.tok[nt] = t; o.rmask[nt] = m; ++nt; }
            }
            o.ntok = nt;
            o.slot = h == 0 ? s0 : s1;
        }
    }
    if (lane < T) { sh.owners[0].tok[lane] = lane; sh.owners[0].rmask[lane] = 1u << k; }
    if (lane == 0) {
        sh.owners[0].slot = prm.P.shared_slot;
        sh.owners[0].ntok = T;
        sh.n_owners = 1 + __popc(b0) + __popc(b1);
    }
    __syncwarp();
}

// ---------------------------------------------------------------- activations to smem
// xs[(n * nb + b) * 36 + j]: pre-scaled activation x_j 2^(23-p_j) of chunk b of
// token n; slots 32..33 hold per-chunk constants: Q2/Q3_32: C = sum x_j 2^(23-p_j),
// X = sum x_j;
// Q3_S256: C'lo, C'hi = sum over the half of x_j (2^(23-p_j) + 4)  (the +4 folds
// the min -4*S of the sub-block into the constant).  Run by the consumer threads.
template <int FMT>
__device__ void stage_activations(const uint16_t* src, size_t tok_stride, int ntok, int K, float* xs,
                                  int first = 0, int nthreads = kConsumers, bool coherent = false) {
    const int nb = K / 32;
    for (int idx = (int)threadIdx.x - first; idx < ntok * nb; idx += nthreads) {
        const int n = idx / nb, b = idx - n * nb;
        const uint4* p = reinterpret_cast<const uint4*>(src + (size_t)n * tok_stride + 32 * b);
        float v[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 w = coherent ? __ldcg(p + q) : __ldg(p + q);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[8 * q + 2 * h] = bf16lo(ww[h]);
                v[8 * q + 2 * h + 1] = bf16hi(ww[h]);
            }
        }
        float* dst = xs + (size_t)idx * kXStride;
        float vp[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) vp[j] = v[j] * (float)(1u << (23 - code_pos<FMT>(j)));   // exact
#pragma unroll
        for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(vp[j], vp[j + 1], vp[j + 2], vp[j + 3]);
        // constants from fp32 partial sums per magic position (few terms each),
        // combined in double: sum_j x_j 2^(23-p_j) (+ 4 x_j for Q3_S256)
        float part[2][10];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 10; ++c) part[h][c] = 0.f;
        float xs0 = 0.f, xs1 = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int c = code_pos<FMT>(j) - 13;       // 0..9
            const int h = (FMT == MOE_Q3_S256 && j >= 16) ? 1 : 0;
            part[h][c] += v[j];
            if (j < 16) xs0 += v[j]; else xs1 += v[j];
        }
        double c0 = 0.0, c1 = 0.0;
#pragma unroll
        for (int c = 0; c < 10; ++c) {
            c0 += (double)part[0][c] * (double)(1u << (10 - c));
            c1 += (double)part[1][c] * (double)(1u << (10 - c));
        }
        if constexpr (FMT == MOE_Q3_S256) {
            c0 += 4.0 * (double)xs0;
            c1 += 4.0 * (double)xs1;
        } else {
            c1 = (double)xs0 + (double)xs1;
        }
        dst[32] = (float)c0;
        dst[33] = (float)c1;
    }
}

// ---------------------------------------------------------------- one chunk, R rows
// cw[r]: the chunk's code words of row r; sa/sb: Q2/Q3_32 (s, m), Q3_S256 (S_lo, S_hi).
// xc[t]: the chunk's activations of the t-th served token.
template <int FMT, int NT, int R>
MOE_DEVINL void chunk_rows(const uint32_t (&cw)[R][3], const float (&sa)[R], const float (&sb)[R],
                           const float* const (&xc)[NT], float (&res)[R][NT]) {
    constexpr int H = (FMT == MOE_Q3_S256) ? 2 : 1;
    const uint32_t one = opaque_one();
    // NC independent accumulator chains per (row, token, half) (even and odd code
    // pairs when few tokens leave registers to spare): shorter FMA dependency chains
    constexpr int NC = NT <= 2 ? 2 : 1;
    float2 acc[R][NT][H][NC];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
                for (int c = 0; c < NC; ++c) acc[r][t][h][c] = make_float2(0.f, 0.f);
    static_for<0, 4>([&](auto SC) {
        constexpr int sc = decltype(SC)::value;
        float xv[NT][8];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float4 a = *reinterpret_cast<const float4*>(xc[t] + 8 * sc);
            const float4 b = *reinterpret_cast<const float4*>(xc[t] + 8 * sc + 4);
            xv[t][0] = a.x; xv[t][1] = a.y; xv[t][2] = a.z; xv[t][3] = a.w;
            xv[t][4] = b.x; xv[t][5] = b.y; xv[t][6] = b.z; xv[t][7] = b.w;
        }
        static_for<0, R>([&](auto RR) {
            constexpr int r = decltype(RR)::value;
            static_for<0, 4>([&](auto II) {
                constexpr int i = 2 * decltype(II)::value;
                constexpr int code = 8 * sc + i;
                constexpr int h = (H == 2 && code >= 16) ? 1 : 0;
                constexpr int c2 = decltype(II)::value % NC;
                const float2 f = make_float2(code_c<FMT, code>(cw[r], one), code_c<FMT, code + 1>(cw[r], one));
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    acc[r][t][h][c2] = ffma2(make_float2(xv[t][i], xv[t][i + 1]), f, acc[r][t][h][c2]);
            });
        });
    });
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const float c0 = xc[t][32];
        const float c1 = xc[t][33];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float sum[H];
#pragma unroll
            for (int h = 0; h < H; ++h) {
                sum[h] = acc[r][t][h][0].x + acc[r][t][h][0].y;
                if constexpr (NC == 2) sum[h] += acc[r][t][h][1].x + acc[r][t][h][1].y;
            }
            if constexpr (H == 2) {
                res[r][t] = __fmaf_rn(sa[r], sum[0] - c0, res[r][t]);
                res[r][t] = __fmaf_rn(sb[r], sum[1] - c1, res[r][t]);
            } else {
                res[r][t] = __fmaf_rn(sa[r], sum[0] - c0, __fmaf_rn(sb[r], c1, res[r][t]));
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
        const float2 sm = __half22float2(*reinterpret_cast<const __half2*>(mbase + (size_t)row * Geo<FMT>::meta_row(K) + b * 4));
        sa = sm.x;
        sb = sm.y;
    } else if constexpr (FMT == MOE_Q3_32) {
        const uint32_t* p = reinterpret_cast<const uint32_t*>(cbase + (size_t)row * Geo<FMT>::code_row(K) + b * 12);
        w[0] = p[0]; w[1] = p[1]; w[2] = p[2];
        const float2 sm = __half22float2(*reinterpret_cast<const __half2*>(mbase + (size_t)row * Geo<FMT>::meta_row(K) + b * 4));
        sa = sm.x;
        sb = sm.y;
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

// ---------------------------------------------------------------- item geometry
// The consumers form two teams of eight warps; a team takes every other item
// of the ring, so that one team's per-item tail (reduction, stores, barrier
// waits) overlaps the other team's inner loops.  Within an item a warp is cut
// into G groups of lpr lanes; a group owns one unit (a gate|up feature or a
// pair of down rows) and its lanes split the unit's nb chunks, nb / lpr each.
// G grows (lpr shrinks) until the team's 8*G groups cover the item's units
// in one pass, which keeps every warp busy and the shuffle reductions short.
// Lane gl of group g takes chunk gl + lpr * ((it + g) mod (nb / lpr)) at
// iteration it: the groups of one warp start on different chunks, so their
// code, scale and activation reads fall in different shared-memory banks.
struct Split { int lpr, G, nit; };
MOE_DEVINL Split split_for(int units, int nb) {
    const int want = units / kTeamWarps;      // groups per warp for one pass
    int gp = 1;                               // largest power of two <= want, at most 8
    while (gp < 8 && 2 * gp <= want) gp *= 2;
    int lpr = 32 / gp;
    const int pow2nb = nb & -nb;              // lpr must divide nb
    if (lpr > pow2nb) lpr = pow2nb;
    Split sp;
    sp.lpr = lpr;
    sp.G = 32 / lpr;
    sp.nit = nb / lpr;
    return sp;
}

// ---------------------------------------------------------------- gate | up
// Item = (owner u, features [f0, f0 + rf)); staged as gate rows then up rows.
// A group computes one feature: its gate row and its up row, chunk by chunk,
// the next chunk's codes read from shared memory while this one is computed.
template <int FMT, int NT>
__device__ void gateup_item(const DecodeParams& prm, const Owner& o, int u, int f0, int rf, const uint8_t* stage,
                            const float* xs, int wt) {
    const int lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F;
    const int nb = D / 32;
    const Split sp = split_for(rf, nb);
    const int lpr = sp.lpr, G = sp.G, nit = sp.nit, group = lane / lpr, gl = lane % lpr;
    const uint32_t cr = Geo<FMT>::code_row(D), mr = Geo<FMT>::meta_row(D);
    const uint32_t half = (uint32_t)Geo<FMT>::row_bytes(D) * rf;   // gate rows then up rows
    const uint8_t* gc = stage;
    const uint8_t* gm = stage + cr * rf;
    const uint8_t* gd = stage + (cr + mr) * rf;
    const uint8_t* uc = stage + half;
    const uint8_t* um = uc + cr * rf;
    const uint8_t* ud = uc + (cr + mr) * rf;
    const float* xt[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) xt[t] = xs + (size_t)o.tok[t] * nb * kXStride;
    for (int base = wt * G; base < rf; base += kTeamWarps * G) {
        const int fq = base + group;
        const bool act = fq < rf;
        const int fl = act ? fq : rf - 1;      // idle groups recompute a valid feature, unstored
        float res[2][NT];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t) res[r][t] = 0.f;
        int c = group % nit;
        int b = gl + lpr * c;
        uint32_t cw[2][3];
        float sa[2], sb[2];
        smem_chunk<FMT>(gc, gm, gd, fl, D, b, cw[0], sa[0], sb[0]);
        smem_chunk<FMT>(uc, um, ud, fl, D, b, cw[1], sa[1], sb[1]);
        for (int it = 0; it < nit; ++it) {
            c = c + 1 == nit ? 0 : c + 1;
            const int bn = gl + lpr * c;       // next chunk (wraps to the first on the last pass: unused)
            uint32_t ncw[2][3];
            float nsa[2], nsb[2];
            smem_chunk<FMT>(gc, gm, gd, fl, D, bn, ncw[0], nsa[0], nsb[0]);
            smem_chunk<FMT>(uc, um, ud, fl, D, bn, ncw[1], nsa[1], nsb[1]);
            const float* xc[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) xc[t] = xt[t] + (size_t)b * kXStride;
            chunk_rows<FMT, NT, 2>(cw, sa, sb, xc, res);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                cw[r][0] = ncw[r][0]; cw[r][1] = ncw[r][1]; cw[r][2] = ncw[r][2];
                sa[r] = nsa[r]; sb[r] = nsb[r];
            }
            b = bn;
        }
        for (int off = lpr >> 1; off >= 1; off >>= 1)
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int t = 0; t < NT; ++t) res[r][t] += __shfl_xor_sync(0xffffffffu, res[r][t], off);
        if (act && gl == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                prm.hbuf[((size_t)u * kDecodeMaxT + t) * F + f0 + fl] = f32_to_bf16_rne(silu_f(res[0][t]) * res[1][t]);
        }
    }
}

// ---------------------------------------------------------------- down
// Item = (owner u, rows [d0, d0 + rd)) of Wd; a group computes two rows.
template <int FMT, int NT>
__device__ void down_item(const DecodeParams& prm, const Owner& o, int d0, int rd, const uint8_t* stage,
                          const float* hs, int wt) {
    const int lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F, k = prm.k;
    const int nb = F / 32;
    const int pairs = rd / 2;
    const Split sp = split_for(pairs, nb);
    const int lpr = sp.lpr, G = sp.G, nit = sp.nit, group = lane / lpr, gl = lane % lpr;
    const uint32_t cr = Geo<FMT>::code_row(F), mr = Geo<FMT>::meta_row(F);
    const uint8_t* dc = stage;
    const uint8_t* dm = stage + cr * rd;
    const uint8_t* dd = stage + (cr + mr) * rd;
    for (int base = wt * G; base < pairs; base += kTeamWarps * G) {
        const int qq = base + group;
        const bool act = qq < pairs;
        const int rl = 2 * (act ? qq : pairs - 1);
        float res[2][NT];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t) res[r][t] = 0.f;
        int c = group % nit;
        int b = gl + lpr * c;
        uint32_t cw[2][3];
        float sa[2], sb[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) smem_chunk<FMT>(dc, dm, dd, rl + r, F, b, cw[r], sa[r], sb[r]);
        for (int it = 0; it < nit; ++it) {
            c = c + 1 == nit ? 0 : c + 1;
            const int bn = gl + lpr * c;
            uint32_t ncw[2][3];
            float nsa[2], nsb[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) smem_chunk<FMT>(dc, dm, dd, rl + r, F, bn, ncw[r], nsa[r], nsb[r]);
            const float* xc[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) xc[t] = hs + ((size_t)t * nb + b) * kXStride;
            chunk_rows<FMT, NT, 2>(cw, sa, sb, xc, res);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                cw[r][0] = ncw[r][0]; cw[r][1] = ncw[r][1]; cw[r][2] = ncw[r][2];
                sa[r] = nsa[r]; sb[r] = nsb[r];
            }
            b = bn;
        }
        for (int off = lpr >> 1; off >= 1; off >>= 1)
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int t = 0; t < NT; ++t) res[r][t] += __shfl_xor_sync(0xffffffffu, res[r][t], off);
        if (act && gl == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float2 v = make_float2(res[0][t], res[1][t]);
                uint32_t m = o.rmask[t];
                while (m) {
                    const int r = __ffs(m) - 1;
                    m &= m - 1;
                    *reinterpret_cast<float2*>(prm.yrows + ((size_t)o.tok[t] * (k + 1) + r) * D + d0 + rl) = v;
                }
            }
        }
    }
}

MOE_DEVINL void st_release_cta(uint32_t* p, uint32_t v) {
    asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(p)), "r"(v) : "memory");
}
MOE_DEVINL uint32_t ld_acquire_cta(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"((uint32_t)__cvta_generic_to_shared(p)) : "memory");
    return v;
}
MOE_DEVINL void red_relaxed_add(uint32_t* p, uint32_t v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
MOE_DEVINL void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Work is balanced by an estimated cost: an item of n weights of an owner
// serving nt tokens costs n / 128 * (4 + 3 (nt - 1)) (a weight served to four
// tokens measured about three times one served to one).  Gate|up items go
// round-robin over the CTAs; each CTA then takes a contiguous range of down
// items such that its gate|up and down costs together approach the average.
MOE_DEVINL int cost_weight(const Shared& sh, int u) { return 4 + 3 * (sh.owners[u].ntok - 1); }
MOE_DEVINL long long warp_sum_ll(long long v) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}
MOE_DEVINL long long warp_incl_scan_ll(long long v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off *= 2) {
        const long long o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}
// One warp computes this CTA's down range [d0, d1) (item_pos order).  Owner u
// has gate|up items from index nfb*(u+1) (owner 0: 0, with 2*nfb half items)
// and down items from nrb*(u+1) (owner 0: 0, 2*nrb half items); gate|up item i
// runs on CTA i mod G.  The cumulative down cost before CTA b is its share of
// all work less the gate|up work of CTAs 0 .. b-1, clamped to [0, total down
// cost]: any such sequence from 0 to the total covers every item (a decrease
// only makes two neighbouring ranges overlap, and an overlapped item is
// computed twice with identical results).
MOE_DEVINL void down_range_warp(const Shared& sh, int b, int G, int nfb, int rf, int D, int nrb, int rd, int F,
                                int& d0, int& d1) {
    constexpr int H = (kMaxPairs + 31) / 32;   // owners per lane: u = lane + 32 h
    const int lane = threadIdx.x & 31, n = sh.n_owners;
    auto below = [&](int m, int cb) {          // #{i < m : i mod G < cb}
        const unsigned q = (unsigned)m / (unsigned)G, r = (unsigned)m % (unsigned)G;
        return (long long)q * cb + (long long)(r < (unsigned)cb ? r : (unsigned)cb);
    };
    long long gu_all = 0, gu_b0 = 0, gu_b1 = 0, dn_part[H];
    int dcost[H], ditems[H];
#pragma unroll
    for (int h = 0; h < H; ++h) {
        const int u = lane + 32 * h;
        dn_part[h] = 0;
        dcost[h] = 1;
        ditems[h] = 0;
        if (u < n) {
            const int w = cost_weight(sh, u);
            const int gi = u == 0 ? 2 * nfb : nfb, gs = u == 0 ? 0 : nfb * (u + 1);
            const long long gc = 2ll * (u == 0 ? rf / 2 : rf) * D / 128 * w;
            gu_all += gc * gi;
            gu_b0 += gc * (below(gs + gi, b) - below(gs, b));
            gu_b1 += gc * (below(gs + gi, b + 1) - below(gs, b + 1));
            ditems[h] = u == 0 ? 2 * nrb : nrb;
            dcost[h] = (u == 0 ? rd / 2 : rd) * F / 128 * w;
            dn_part[h] = (long long)dcost[h] * ditems[h];
        }
    }
    gu_all = warp_sum_ll(gu_all);
    gu_b0 = warp_sum_ll(gu_b0);
    gu_b1 = warp_sum_ll(gu_b1);
    // exclusive prefix of the down costs over owners 0 .. n-1, 32 owners a pass
    long long base[H], carry = 0;
#pragma unroll
    for (int h = 0; h < H; ++h) {
        const long long in = warp_incl_scan_ll(dn_part[h]) + carry;
        base[h] = in - dn_part[h];
        carry = __shfl_sync(0xffffffffu, in, 31);
    }
    const long long dn_all = carry;
    const long long all = gu_all + dn_all;
    auto start = [&](int cb, long long gub) -> long long {
        if (cb <= 0) return 0;
        if (cb >= G) return dn_all;
        const long long ds = (all * cb + G - 1) / G - gub;
        return ds < 0 ? 0 : (ds > dn_all ? dn_all : ds);
    };
    auto item_at = [&](long long pos) -> int {
        int idx = -1;
#pragma unroll
        for (int h = 0; h < H; ++h) {
            const int u = lane + 32 * h;
            if (u < n && pos >= base[h] && pos < base[h] + dn_part[h]) {
                const int m = (int)((pos - base[h] + dcost[h] - 1) / dcost[h]);
                idx = (u == 0 ? 0 : nrb * (u + 1)) + (m < ditems[h] ? m : ditems[h]);
            }
        }
        const uint32_t hit = __ballot_sync(0xffffffffu, idx >= 0);
        return hit ? __shfl_sync(0xffffffffu, idx, __ffs(hit) - 1) : (n == 0 ? 0 : nrb * (n + 1));
    };
    d0 = item_at(start(b, gu_b0));
    d1 = item_at(start(b + 1, gu_b1));
}

MOE_DEVINL uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ---------------------------------------------------------------- the fused kernel
// One persistent CTA per SM.  Each CTA takes its gate|up items (round-robin),
// then a contiguous range of down items (balancing the estimated cost of both),
// through one ring of stages.  A down item of owner u waits until every
// gate|up item of u has published its h: a per-owner item counter in ws,
// advanced by a publisher warp that releases each finished item at gpu scope,
// off the computing warps' path.  The down weights stream in meanwhile.  The
// last CTA to finish resets the counters, so every completed call leaves them
// zero.
template <int FMT, int NTMAX>
__global__ void __launch_bounds__(kThreads, 1) decode_ffn_kernel(DecodeParams prm) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ Shared sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F, rf = prm.rf, rd = prm.rd, NS = prm.ns_gu;
    const int nbx = D / 32, nbh = F / 32;
    const size_t xs_bytes = ((size_t)prm.T * nbx * kXStride * 4 + 127) / 128 * 128;
    const size_t hs_floats = ((size_t)kDecodeMaxT * nbh * kXStride + 31) / 32 * 32;   // one per team
    const size_t hs_bytes = kTeams * hs_floats * 4;
    float* xs = reinterpret_cast<float*>(smem);
    float* hs = reinterpret_cast<float*>(smem + xs_bytes);
    uint8_t* stages = smem + xs_bytes + hs_bytes;
    const uint32_t gu_bytes = 2u * Geo<FMT>::row_bytes(D) * rf;
    const uint32_t dn_bytes = (uint32_t)Geo<FMT>::row_bytes(F) * rd;
    const uint32_t stage_bytes = gu_bytes > dn_bytes ? gu_bytes : dn_bytes;
    const int nfb = F / rf, nrb = D / rd;
    uint32_t* done = prm.done;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], kTeamWarps); }
        mbar_init(&sh.range_bar, 1);
        fence_mbar_init();
        for (int tm = 0; tm < kTeams; ++tm) { sh.abort[tm] = 0; sh.team_items[tm] = 0; }
    }
    stage_table(prm, sh);
    __syncthreads();
    pdl_wait();                      // ids come from the router
    // a call on a workspace whose timeout bit is set does no work (every CTA
    // still takes its ticket below, so the counters are left zero); one read,
    // shared by the whole CTA, so that every warp takes the same branch
    __shared__ int dead;
    if (threadIdx.x == 0) dead = timed_out(prm.err) ? 1 : 0;
    __syncthreads();
    if (!dead) {
    // warp 0 resolves the owners and releases the producer and publisher
    // (barrier 1) while the other consumers stage x; the consumers meet at
    // barrier 4 before computing
    if (warp == 0) {
        resolve_owners(prm, sh, blockIdx.x == 0);
        asm volatile("bar.arrive 1, 96;" ::: "memory");
        asm volatile("bar.sync 4, %0;" ::"n"(kConsumers) : "memory");
    } else if (warp < kConsumerWarps) {
        stage_activations<FMT>(prm.x, D, prm.T, D, xs, 32, kConsumers - 32);
        asm volatile("bar.sync 4, %0;" ::"n"(kConsumers) : "memory");
    } else {
        asm volatile("bar.sync 1, 96;" ::: "memory");
    }
    pdl_launch_dependents();
    // gate|up items round-robin over the CTAs (x is staged for every token);
    // down items in contiguous ranges of equal cost (h is re-staged per owner)
    const int n_g = items_of(sh.n_owners, nfb);
    const int ng = n_g > (int)blockIdx.x ? (n_g - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    // the down range is computed by the publisher warp, off the producer's path;
    // the others wait for it only when they reach their first down item
    int d0r = 0, d1r = 0;
    bool have_range = false;
    auto get_range = [&]() -> bool {
        if (!have_range) {
            if (!mbar_wait(&sh.range_bar, 0, prm.err)) return false;
            d0r = sh.d_range[0];
            d1r = sh.d_range[1];
            have_range = true;
        }
        return true;
    };
    if (warp == kPublisherWarp) {    // publisher: the down range, then release finished gate|up items
        {
            int r0, r1;
            down_range_warp(sh, (int)blockIdx.x, (int)gridDim.x, nfb, rf, D, nrb, rd, F, r0, r1);
            if (lane == 0) {
                sh.d_range[0] = r0;
                sh.d_range[1] = r1;
                mbar_arrive(&sh.range_bar);
            }
        }
        if (lane == 0) {
            uint32_t pub[kTeams] = {0u, 0u};
            const uint32_t want[kTeams] = {(uint32_t)((ng + 1) / 2), (uint32_t)(ng / 2)};
            const uint64_t t0 = globaltimer_ns();
            while (pub[0] < want[0] || pub[1] < want[1]) {
                const uint32_t c0 = ld_acquire_cta(&sh.team_items[0]), c1 = ld_acquire_cta(&sh.team_items[1]);
                if (c0 > pub[0] || c1 > pub[1]) {
                    fence_acq_rel_gpu();             // with the relaxed adds below: one release per batch
                    const uint32_t c[kTeams] = {c0, c1};
                    for (int tm = 0; tm < kTeams; ++tm)
                        for (uint32_t n = pub[tm]; n < c[tm]; ++n) {
                            const int j = tm + kTeams * (int)n;
                            red_relaxed_add(done + item_pos(blockIdx.x + j * gridDim.x, nfb, rf).u, 1u);
                        }
                    pub[0] = c0;
                    pub[1] = c1;
                } else {
                    if (timed_out(prm.err) ||
                        *reinterpret_cast<volatile int*>(&sh.abort[0]) || *reinterpret_cast<volatile int*>(&sh.abort[1]))
                        break;
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        atomicOr(prm.err, kErrTimeout);
                        break;
                    }
                    __nanosleep(32);
                }
            }
        }
    } else if (warp == kProducerWarp) {    // producer: gate|up items, then down items
        if (lane == 0) {
            for (int j = 0;; ++j) {
                if (j >= ng && !get_range()) break;
                if (j >= ng + (d1r - d0r)) break;
                const int s = j % NS;
                if (j >= NS && !mbar_wait(&sh.empty[s], ((j / NS) - 1) & 1, prm.err)) break;
                if (*reinterpret_cast<volatile int*>(&sh.abort[0]) | *reinterpret_cast<volatile int*>(&sh.abort[1])) break;
                uint8_t* dst = stages + (size_t)s * stage_bytes;
                if (j < ng) {
                    const ItemPos ip = item_pos(blockIdx.x + j * gridDim.x, nfb, rf);
                    const int slot = sh.owners[ip.u].slot;
                    const uint32_t half = (uint32_t)Geo<FMT>::row_bytes(D) * ip.nrows;
                    mbar_arrive_expect_tx(&sh.full[s], 2 * half);
                    issue_rows<FMT>(planes_of<FMT>(prm.P, slot, 0), ip.row0, ip.nrows, D, dst, &sh.full[s]);
                    issue_rows<FMT>(planes_of<FMT>(prm.P, slot, 1), ip.row0, ip.nrows, D, dst + half, &sh.full[s]);
                } else {
                    const ItemPos ip = item_pos(d0r + (j - ng), nrb, rd);
                    mbar_arrive_expect_tx(&sh.full[s], (uint32_t)Geo<FMT>::row_bytes(F) * ip.nrows);
                    issue_rows<FMT>(planes_of<FMT>(prm.P, sh.owners[ip.u].slot, 2), ip.row0, ip.nrows, F, dst, &sh.full[s]);
                }
            }
        }
    } else {
        // consumer teams: team tm takes items j = tm, tm + 2, ... of the ring
        const int team = warp / kTeamWarps, wt = warp % kTeamWarps;
        const int tl = (int)threadIdx.x - team * kTeamWarps * 32;
        float* hst = hs + (size_t)team * hs_floats;
        bool ok = true;
        int cur = -1;
        uint32_t gu_done = 0;
        for (int j = team;; j += kTeams) {
            if (j >= ng) {
                ok = team_all(team, get_range());     // the same verdict on every thread of the team
                if (!ok) break;
                if (j >= ng + (d1r - d0r)) break;
            }
            const int s = j % NS;
            const uint8_t* st = stages + (size_t)s * stage_bytes;
            if (j < ng) {
                bool got = mbar_wait(&sh.full[s], (j / NS) & 1, prm.err);
                const ItemPos ip = item_pos(blockIdx.x + j * gridDim.x, nfb, rf);
                const int u = ip.u, f0 = ip.row0;
                const Owner& o = sh.owners[u];
                if (got) {
                    if constexpr (NTMAX == 1) {
                        gateup_item<FMT, 1>(prm, o, u, f0, ip.nrows, st, xs, wt);
                    } else {
                        switch (o.ntok) {
                            case 1: gateup_item<FMT, 1>(prm, o, u, f0, ip.nrows, st, xs, wt); break;
                            case 2: gateup_item<FMT, 2>(prm, o, u, f0, ip.nrows, st, xs, wt); break;
                            case 3: gateup_item<FMT, 3>(prm, o, u, f0, ip.nrows, st, xs, wt); break;
                            default: gateup_item<FMT, 4>(prm, o, u, f0, ip.nrows, st, xs, wt); break;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.empty[s]);
                // the team's h stores of this item are done (and the verdict is
                // the team's, so every thread leaves the loop together): publish
                ok = team_all(team, got);
                if (!ok) break;
                ++gu_done;
                if (tl == 0) st_release_cta(&sh.team_items[team], gu_done);
            } else {
                const ItemPos ip = item_pos(d0r + (j - ng), nrb, rd);
                const int u = ip.u, r0 = ip.row0;
                const Owner& o = sh.owners[u];
                if (u != cur) {
                    team_sync(team);                    // the team is done reading hst
                    bool waited = true;
                    if (tl == 0) {
                        const uint32_t target = (uint32_t)(u == 0 ? 2 * nfb : nfb);   // items of owner u
                        const uint64_t t0 = globaltimer_ns();
                        while (ld_acquire(done + u) < target) {
                            if (timed_out(prm.err) || globaltimer_ns() - t0 > kWaitLimitNs) {
                                atomicOr(prm.err, kErrTimeout);
                                waited = false;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    ok = team_all(team, waited);
                    if (!ok) break;
                    stage_activations<FMT>(prm.hbuf + (size_t)u * kDecodeMaxT * F, F, o.ntok, F, hst,
                                           team * kTeamWarps * 32, kTeamWarps * 32, true);
                    team_sync(team);
                    cur = u;
                }
                const bool got = mbar_wait(&sh.full[s], (j / NS) & 1, prm.err);
                if (got) {
                    if constexpr (NTMAX == 1) {
                        down_item<FMT, 1>(prm, o, r0, ip.nrows, st, hst, wt);
                    } else {
                        switch (o.ntok) {
                            case 1: down_item<FMT, 1>(prm, o, r0, ip.nrows, st, hst, wt); break;
                            case 2: down_item<FMT, 2>(prm, o, r0, ip.nrows, st, hst, wt); break;
                            case 3: down_item<FMT, 3>(prm, o, r0, ip.nrows, st, hst, wt); break;
                            default: down_item<FMT, 4>(prm, o, r0, ip.nrows, st, hst, wt); break;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.empty[s]);
                ok = team_all(team, got);
                if (!ok) break;
            }
        }
        if (!ok && tl == 0) sh.abort[team] = 1;
    }
    }   // !dead
    // last CTA out resets the per-owner counters for the next call
    // (acq_rel ticket: this CTA's counter updates, ordered before it by the
    // barrier, precede the reset; the last CTA sees every other CTA's)
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t ticket;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(ticket) : "l"(done + kMaxPairs) : "memory");
        if (ticket == gridDim.x - 1) {
            for (int u = 0; u < kMaxPairs; ++u) done[u] = 0u;
            done[kMaxPairs] = 0u;
        }
    }
}

template <int FMT, int NTMAX>
moe_status launch_fmt(DecodeParams prm, cudaStream_t s) {
    const int T = prm.T, D = prm.P.D, F = prm.P.F;
    const size_t xs_bytes = ((size_t)T * (D / 32) * kXStride * 4 + 127) / 128 * 128;
    const size_t hs_bytes = kTeams * (((size_t)kDecodeMaxT * (F / 32) * kXStride + 31) / 32 * 32) * 4;
    // gate|up items of rf features, down items of rd rows, one ring of up to 4
    // stages (~3-4 items in flight per SM cover the copy latency)
    int rf = 16, rd = 128;
    const size_t budget = 216 * 1024;
    auto stage_of = [&](int rf_, int rd_) {
        const size_t a = 2 * (size_t)Geo<FMT>::row_bytes(D) * rf_, b = (size_t)Geo<FMT>::row_bytes(F) * rd_;
        return a > b ? a : b;
    };
    while (rf > 2 && xs_bytes + hs_bytes + 2 * stage_of(rf, rd) > budget) rf /= 2;
    while (rd > 16 && (size_t)Geo<FMT>::row_bytes(F) * rd > 2 * (size_t)Geo<FMT>::row_bytes(D) * rf) rd /= 2;
    int ns = 4;
    while (ns > 2 && xs_bytes + hs_bytes + ns * stage_of(rf, rd) > budget) --ns;
    prm.rf = rf;
    prm.rd = rd;
    prm.ns_gu = prm.ns_dn = ns;
    const size_t smem = xs_bytes + hs_bytes + ns * stage_of(rf, rd);
    if (smem > kSmemBudget || F % rf || D % rd || rf < 2 || rd < 2) return MOE_ERR_UNSUPPORTED;
    // every bulk copy (full and half items) must be a multiple of 16 bytes
    auto ok16 = [](int K, int n) {
        return ((size_t)Geo<FMT>::code_row(K) * n) % 16 == 0 && ((size_t)Geo<FMT>::meta_row(K) * n) % 16 == 0 &&
               ((size_t)Geo<FMT>::d_row(K) * n) % 16 == 0;
    };
    if (!ok16(D, rf) || !ok16(D, rf / 2) || !ok16(F, rd) || !ok16(F, rd / 2)) return MOE_ERR_UNSUPPORTED;
    static std::atomic<uint64_t> attr_done{0};
    if (!once_per_device(attr_done, [] {
            return cudaFuncSetAttribute(decode_ffn_kernel<FMT, NTMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kSmemBudget) == cudaSuccess;
        }))
        return MOE_ERR_CUDA;
    cudaError_t e = launch_pdl(decode_ffn_kernel<FMT, NTMAX>, dim3(device_sm_count()), dim3(kThreads), smem, s, prm);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

// ws layout: [0,4) reserved, [4,8) device error word, [64, 64 + 4*(kMaxPairs+1))
// completion counters (zero before the first call; every completed call leaves
// them zero), [1024, ...) h buffer.
size_t decode_workspace_bytes(int T, int D, int F, int k) {
    (void)D; (void)T; (void)k;
    return 1024 + (size_t)kMaxPairs * kDecodeMaxT * F * sizeof(uint16_t);
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
    prm.done = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 64);
    prm.hbuf = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(ws) + 1024);
    const bool one = (T == 1);
    switch (P.fmt) {
        case MOE_Q2_32: return one ? launch_fmt<MOE_Q2_32, 1>(prm, s) : launch_fmt<MOE_Q2_32, 4>(prm, s);
        case MOE_Q3_32: return one ? launch_fmt<MOE_Q3_32, 1>(prm, s) : launch_fmt<MOE_Q3_32, 4>(prm, s);
        default: return one ? launch_fmt<MOE_Q3_S256, 1>(prm, s) : launch_fmt<MOE_Q3_S256, 4>(prm, s);
    }
}

}  // namespace moe
