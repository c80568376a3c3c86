// prefill.cu — expert pass for chunks of many tokens (T > 4): a deterministic
// tokens-by-expert permute, then two grouped GEMMs on the 5th-generation tensor
// cores (tcgen05) whose weight operand is dequantised from the 2-/3-bit blocks
// on the fly, straight into tensor memory.
//
// The pages: prefill runs in chunks, with expert transfers overlapped with GPU
// compute (greenbean-ai "Strata 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next" §三);
// 10 routed + 1 shared experts per token (wiselychen RTX 5090 report,
// "30 秒定位"); weights are 2-3.5 bit block-quantised (wiselychen report §1).
//
// Rows.  Every resident (token, rank) pair and every token's shared-expert
// evaluation is one row; rows are grouped by expert (routed experts in id
// order, tokens ascending within an expert), then the T shared rows.
//   GEMM 1 (gate|up): per tile of 64 features x up to 128 rows of one group,
//     one M = 128 accumulator holds Wg x (lanes 0..63) and Wu x (lanes
//     64..127) in TMEM; epilogue h = bf16(silu(Wg x) * (Wu x))
//   GEMM 2 (down): per tile of 128 outputs x up to 128 rows, acc = Wd h;
//     epilogue y = bf16(acc) into the expert_out rows
// Both are "swap-AB": the weights are the M = 128 operand (A, in tensor
// memory), the rows are N (B, in shared memory).
//
// Operand type.  The MMAs run kind::f16 with fp16 A and B.  Every weight is
// the exact weight rounded once to fp16 (dequant.cuh) — finer than a bf16
// weight.  The bf16 activations convert to fp16 exactly inside the fp16 range;
// an activation of magnitude >= 65520 (x or h) sets kErrRange in the error word.
//
// K order.  Inside every group of 16 consecutive K indices the operands use
// the order (0, 8, 1, 9, ..., 7, 15): one 32-bit word of A then holds the
// weight pair (i, i + 8), which the block formats deliver in the same word at
// the same bit offset of both halves.  The rows of x are gathered into group
// order and converted (gather_f16p_kernel), so that both GEMMs read their row
// operand as contiguous 2D TMA boxes; h (down) is written in that order by the
// gate|up epilogue.
#include <cuda.h>            // CUtensorMap types; the encoder is fetched at run time
#include <cuda_fp16.h>

#include "common.cuh"
#include "dequant.cuh"
#include "kernels.cuh"
#include "once.cuh"
#include "sync.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

constexpr int kChunk = 256;            // tokens per plan chunk
constexpr int kGatherThreads = 64;     // threads per row of the x gather (D / 16 groups of 16 elements)
constexpr int kMaxE = 1024;
constexpr int kN1 = 128;               // max rows per gate|up tile
constexpr int kN2 = 128;               // max rows per down tile
constexpr int kGateFeat = 128;         // gate|up tile: 128 gate + the same 128 up features
constexpr int kDownRows = 256;         // down tile: 256 outputs
constexpr int kKAlign = 128;           // D and F are multiples of this
constexpr int kDqWarps = 16;           // dequantisation warps: two halves of 256 threads (one per weight row)
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = kDqWarps + kEpiWarps;
constexpr int kGatherWarp = kTmaWarp + 1;
constexpr int kMmaWarp = kGatherWarp + 1;
constexpr int kGemmThreads = (kMmaWarp + 1) * 32;

// ---------------------------------------------------------------- workspace
struct PrefillWs {
    int32_t* hist;        // [nchunk][E]: hits of expert e in the chunk, then the chunk's base row
    int32_t* miss_hist;   // [nchunk]: misses in the chunk, then the chunk's base index
    int32_t* meta;        // [0] rows of routed groups, [1] tiles1, [2] tiles2
    int4* tiles1;         // (group row0, rows, m0, slot)
    int4* tiles2;
    int32_t* perm;        // [rows] token of each row
    uint16_t* xg;         // [rows][D] fp16, K-permuted: x of each row's token
    uint16_t* h;          // [rows][F] fp16, K-permuted
    uint32_t* err;
};

inline size_t align256(size_t n) { return (n + 255) / 256 * 256; }

struct WsSizes {
    size_t hist, miss, meta, t1, t2, perm, xg, h, total;
    size_t max_t1, max_t2;
};

inline WsSizes ws_sizes(int T, int D, int F, int E, int k) {
    const int nchunk = (T + kChunk - 1) / kChunk;
    const size_t rows = (size_t)T * (k + 1);
    WsSizes s;
    // bound on sum over groups of ceil(n / N): rows / N + (number of groups)
    s.max_t1 = (rows / kN1 + (size_t)E + 2) * (F / kGateFeat);
    s.max_t2 = (rows / kN2 + (size_t)E + 2) * (D / kDownRows);
    s.hist = align256((size_t)nchunk * E * 4);
    s.miss = align256((size_t)nchunk * 4);
    s.meta = 256;
    s.t1 = align256(s.max_t1 * sizeof(int4));
    s.t2 = align256(s.max_t2 * sizeof(int4));
    s.perm = align256(rows * 4);
    s.xg = align256(rows * D * 2);
    s.h = align256(rows * F * 2);
    s.total = 1024 + s.hist + s.miss + s.meta + s.t1 + s.t2 + s.perm + s.xg + s.h;
    return s;
}

inline PrefillWs carve(void* ws, int T, int D, int F, int E, int k) {
    const WsSizes s = ws_sizes(T, D, F, E, k);
    char* p = reinterpret_cast<char*>(ws);
    PrefillWs w;
    w.err = reinterpret_cast<uint32_t*>(p + 4);
    p += 1024;   // the first 1024 bytes follow the decode path's layout (error word, counters)
    w.hist = reinterpret_cast<int32_t*>(p); p += s.hist;
    w.miss_hist = reinterpret_cast<int32_t*>(p); p += s.miss;
    w.meta = reinterpret_cast<int32_t*>(p); p += s.meta;
    w.tiles1 = reinterpret_cast<int4*>(p); p += s.t1;
    w.tiles2 = reinterpret_cast<int4*>(p); p += s.t2;
    w.perm = reinterpret_cast<int32_t*>(p); p += s.perm;
    w.xg = reinterpret_cast<uint16_t*>(p); p += s.xg;
    w.h = reinterpret_cast<uint16_t*>(p);
    return w;
}

// ---------------------------------------------------------------- plan
struct PlanArgs {
    const int32_t* ids;
    const int32_t* slot_table;
    int T, k, E, n_slots, shared_slot, F, D;
    PrefillWs w;
    int32_t* rowmap;      // [T][k+1]
    int32_t* miss_list;
    int32_t* miss_count;
};

__device__ __forceinline__ int plan_slot(const PlanArgs& a, int e) {
    const int s = (e >= 0 && e < a.E) ? __ldg(a.slot_table + e) : -1;
    return (s < 0 || s >= a.n_slots) ? -1 : s;
}

// Per chunk of 256 tokens: a bitmask of the chunk's tokens for every expert
// (bit t set when token t of the chunk selected the expert and it is resident).
__device__ void chunk_masks(const PlanArgs& a, int chunk, uint32_t (*mask)[kChunk / 32], int& my_miss,
                            int (&eid)[kMaxTopK], uint32_t& hit) {
    for (int i = threadIdx.x; i < a.E * (kChunk / 32); i += blockDim.x) mask[i / (kChunk / 32)][i % (kChunk / 32)] = 0;
    const int t = chunk * kChunk + threadIdx.x;
    my_miss = 0;
    hit = 0;
    // the token's ids, then their slots: all loads of one kind in flight together
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) eid[r] = (t < a.T && r < a.k) ? __ldg(a.ids + (size_t)t * a.k + r) : -1;
    int sl[kMaxTopK];
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) sl[r] = r < a.k ? plan_slot(a, eid[r]) : -1;
    __syncthreads();
    if (t < a.T) {
#pragma unroll
        for (int r = 0; r < kMaxTopK; ++r) {
            if (r >= a.k) break;
            if (sl[r] >= 0) {
                atomicOr(&mask[eid[r]][threadIdx.x >> 5], 1u << (threadIdx.x & 31));
                hit |= 1u << r;
            } else {
                ++my_miss;
            }
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kChunk) plan_count_kernel(PlanArgs a) {
    __shared__ uint32_t mask[kMaxE][kChunk / 32];
    __shared__ int wsum[kChunk / 32];
    pdl_wait();
    int my_miss;
    int eid[kMaxTopK];
    uint32_t hit;
    chunk_masks(a, blockIdx.x, mask, my_miss, eid, hit);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kChunk / 32; ++w) c += __popc(mask[e][w]);
        a.w.hist[(size_t)blockIdx.x * a.E + e] = c;
    }
    int v = my_miss;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        int s = 0;
        for (int w = 0; w < kChunk / 32; ++w) s += wsum[w];
        a.w.miss_hist[blockIdx.x] = s;
    }
}

// One CTA: expert offsets, per-chunk bases, miss bases and the two tile lists.
// Exclusive prefix sum of v over the 1024 threads of the block; *total gets the
// block's sum.  Every thread calls it.
MOE_DEVINL int block_exscan1024(int v, int* total) {
    __shared__ int wsum[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    if (w == 0) {
        int t = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        wsum[lane] = t;
    }
    __syncthreads();
    const int r = (w > 0 ? wsum[w - 1] : 0) + x - v;
    *total = wsum[31];
    __syncthreads();                              // wsum is reused by the next call
    return r;
}

// Largest g in [0, last] with off[g] <= i (off non-decreasing, off[0] = 0 <= i).
MOE_DEVINL int group_of(const int* off, int last, int i) {
    int lo = 0, hi = last;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// One block of 1024 threads: groups' totals, row offsets and tile offsets (block
// scans over the E routed groups and the shared group E), the misses' chunk
// offsets, every chunk's base row per expert, and the two tile lists (group, row
// tile, then weight-row tile, the fastest index), one entry per thread in turn.
__global__ void __launch_bounds__(1024) plan_scan_kernel(PlanArgs a) {
    __shared__ int tot[kMaxE];
    __shared__ int off[kMaxE + 1];
    __shared__ int t1off[kMaxE + 2];
    __shared__ int t2off[kMaxE + 2];
    __shared__ int gslot[kMaxE + 1];
    pdl_wait();
    const int nchunk = (a.T + kChunk - 1) / kChunk;
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) {
        if (e == a.E) { gslot[e] = a.shared_slot; continue; }
        int run = 0;
#pragma unroll 8
        for (int c = 0; c < nchunk; ++c) run += a.w.hist[(size_t)c * a.E + e];
        tot[e] = run;
        gslot[e] = plan_slot(a, e);
    }
    __syncthreads();
    // groups 0..E-1 routed (rows tot[e]), group E the shared expert (T rows)
    int c_rows = 0, c_t1 = 0, c_t2 = 0;
    for (int base = 0; base <= a.E; base += 1024) {
        const int g = base + (int)threadIdx.x;
        const int n = g < a.E ? tot[g] : (g == a.E ? a.T : 0);
        int s_rows, s_t1, s_t2;
        const int x_rows = block_exscan1024(g < a.E ? n : 0, &s_rows);
        const int x_t1 = block_exscan1024((n + kN1 - 1) / kN1, &s_t1);
        const int x_t2 = block_exscan1024((n + kN2 - 1) / kN2, &s_t2);
        if (g <= a.E) {
            off[g] = c_rows + x_rows;
            t1off[g] = c_t1 + x_t1;
            t2off[g] = c_t2 + x_t2;
        }
        c_rows += s_rows;
        c_t1 += s_t1;
        c_t2 += s_t2;
    }
    if (threadIdx.x == 0) {
        t1off[a.E + 1] = c_t1;
        t2off[a.E + 1] = c_t2;
        a.w.meta[0] = c_rows;
        a.w.meta[1] = c_t1 * (a.F / kGateFeat);
        a.w.meta[2] = c_t2 * (a.D / kDownRows);
    }
    // misses: exclusive scan over chunks (token-major order)
    int c_miss = 0;
    for (int base = 0; base < nchunk; base += 1024) {
        const int c = base + (int)threadIdx.x;
        int s_miss;
        const int v = c < nchunk ? a.w.miss_hist[c] : 0;
        const int x_miss = block_exscan1024(v, &s_miss);
        if (c < nchunk) a.w.miss_hist[c] = c_miss + x_miss;
        c_miss += s_miss;
    }
    if (threadIdx.x == 0) a.miss_count[0] = c_miss;
    __syncthreads();
    // per-chunk base rows of every expert: eight chunks' counts loaded before their
    // base rows are written back
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = off[e];
        for (int c0 = 0; c0 < nchunk; c0 += 8) {
            int v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = c0 + i < nchunk ? a.w.hist[(size_t)(c0 + i) * a.E + e] : 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (c0 + i < nchunk) {
                    a.w.hist[(size_t)(c0 + i) * a.E + e] = run;
                    run += v[i];
                }
            }
        }
    }
    // tile lists
    const int mt1 = a.F / kGateFeat, mt2 = a.D / kDownRows;
    const int n1 = c_t1 * mt1, n2 = c_t2 * mt2;
    for (int i = threadIdx.x; i < n1 + n2; i += blockDim.x) {
        const bool first_list = i < n1;
        const int ii = first_list ? i : i - n1;
        const int mt = first_list ? mt1 : mt2;
        const int tile = ii / mt, m = ii % mt;
        const int* toff = first_list ? t1off : t2off;
        const int g = group_of(toff, a.E, tile);
        const int n = g < a.E ? tot[g] : a.T;
        const int j = tile - toff[g];
        const int nr = first_list ? kN1 : kN2;
        const int4 td = make_int4(off[g] + j * nr, min(nr, n - j * nr), m * (first_list ? kGateFeat : kDownRows), gslot[g]);
        if (first_list) a.w.tiles1[ii] = td;
        else a.w.tiles2[ii] = td;
    }
}

// Rows of every hit (stable: tokens ascending within an expert), the row map,
// the shared rows and the miss list (token-major, rank order).
__global__ void __launch_bounds__(kChunk) plan_scatter_kernel(PlanArgs a) {
    __shared__ uint32_t mask[kMaxE][kChunk / 32];
    __shared__ int wsum[kChunk / 32];
    pdl_wait();
    int my_miss;
    int eid[kMaxTopK];
    uint32_t hit;
    chunk_masks(a, blockIdx.x, mask, my_miss, eid, hit);
    // exclusive scan of misses over the chunk's threads
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int v = my_miss;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    int wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += wsum[w];
    int mpos = a.w.miss_hist[blockIdx.x] + wbase + v - my_miss;
    const int t = blockIdx.x * kChunk + threadIdx.x;
    if (t >= a.T) return;
    const int S = a.w.meta[0];
    const int k = a.k;
    // the chunk's base row of each hit expert: all loads in flight together
    int hb[kMaxTopK];
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) hb[r] = (hit >> r) & 1u ? a.w.hist[(size_t)blockIdx.x * a.E + eid[r]] : 0;
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) {
        if (r >= k) break;
        const int e = eid[r];
        if ((hit >> r) & 1u) {
            int below = 0;
            const int wi = threadIdx.x >> 5;
            for (int w = 0; w < wi; ++w) below += __popc(mask[e][w]);
            below += __popc(mask[e][wi] & ((1u << (threadIdx.x & 31)) - 1u));
            const int row = hb[r] + below;
            a.w.perm[row] = t;
            a.rowmap[(size_t)t * (k + 1) + r] = row;
        } else {
            a.rowmap[(size_t)t * (k + 1) + r] = -1;
            a.miss_list[3 * mpos + 0] = t;
            a.miss_list[3 * mpos + 1] = r;
            a.miss_list[3 * mpos + 2] = e;
            ++mpos;
        }
    }
    a.w.perm[S + t] = t;
    a.rowmap[(size_t)t * (k + 1) + k] = S + t;
}

// ---------------------------------------------------------------- x rows -> fp16, group order, K-permuted
MOE_DEVINL uint32_t bf16_half(uint32_t w, int hi) { return hi ? (w & 0xffff0000u) : (w << 16); }

// xg[row] = x[perm[row]] in fp16 and K order: one thread per 16-element group,
// out word i = (x[i], x[i + 8]).  Rows: the routed rows, then the T shared rows.
__global__ void __launch_bounds__(kGatherThreads) gather_f16p_kernel(const uint16_t* __restrict__ x,
                                                                      const int32_t* __restrict__ perm,
                                                                      const int32_t* __restrict__ meta, int T, int D,
                                                                      uint16_t* __restrict__ xg, uint32_t* err) {
    // one block per row (rows past the routed groups + the shared group return)
    pdl_wait();
    const int row = blockIdx.x;
    if (row >= __ldg(meta) + T) return;
    const uint16_t* xr = x + (size_t)__ldg(perm + row) * D;
    uint16_t* dr = xg + (size_t)row * D;
    bool bad = false;
    for (int gc = threadIdx.x; gc < D / 16; gc += kGatherThreads) {
        const uint4* src = reinterpret_cast<const uint4*>(xr + gc * 16);
        const uint4 a = __ldg(src), b = __ldg(src + 1);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float lo = __uint_as_float(bf16_half(aw[i >> 1], i & 1));
            const float hi = __uint_as_float(bf16_half(bw[i >> 1], i & 1));
            bad |= !(fabsf(lo) < 65520.f) || !(fabsf(hi) < 65520.f);
            o[i] = pack_f16x2(lo, hi);
        }
        uint4* dst = reinterpret_cast<uint4*>(dr + gc * 16);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    if (bad) atomicOr(err, kErrRange);
}

// Two fp16 values (a pair word) to two e4m3 bytes, rounded to nearest even and
// saturated to the finite range: the low half to bits 0..7.
MOE_DEVINL uint32_t e4m3x2_of_f16x2(uint32_t h2) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(d) : "r"(h2));
    return d;
}
// Two fp32 values to two e4m3 bytes (nearest even, saturated): lo in bits 0..7.
MOE_DEVINL uint32_t e4m3x2_of_f32(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// The e4m3 variant: x rows in group order as e4m3 bytes, K-permuted the same way
// (bytes 2i, 2i + 1 of a 16-group = elements i, i + 8), rounded to nearest even
// and saturated; |x| >= 448 sets the range bit.
__global__ void __launch_bounds__(kGatherThreads) gather_f8p_kernel(const uint16_t* __restrict__ x,
                                                                     const int32_t* __restrict__ perm,
                                                                     const int32_t* __restrict__ meta, int T, int D,
                                                                     uint8_t* __restrict__ xg, uint32_t* err) {
    pdl_wait();
    const int row = blockIdx.x;
    if (row >= __ldg(meta) + T) return;
    const uint16_t* xr = x + (size_t)__ldg(perm + row) * D;
    uint8_t* dr = xg + (size_t)row * D;
    bool bad = false;
    for (int gc = threadIdx.x; gc < D / 16; gc += kGatherThreads) {
        const uint4* src = reinterpret_cast<const uint4*>(xr + gc * 16);
        const uint4 a = __ldg(src), b = __ldg(src + 1);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
        uint32_t o[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float lo = __uint_as_float(bf16_half(aw[i >> 1], i & 1));
            const float hi = __uint_as_float(bf16_half(bw[i >> 1], i & 1));
            bad |= !(fabsf(lo) < 448.f) || !(fabsf(hi) < 448.f);
            o[i >> 1] |= e4m3x2_of_f32(lo, hi) << (16 * (i & 1));
        }
        *reinterpret_cast<uint4*>(dr + gc * 16) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (bad) atomicOr(err, kErrRange);
}

// ---------------------------------------------------------------- tcgen05 / TMA helpers
MOE_DEVINL uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3ffffu) >> 4);        // start address
    d |= (uint64_t)1 << 16;                           // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024 >> 4) << 32;                 // stride byte offset: 8-row groups
    d |= (uint64_t)1 << 46;                           // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                           // 128-byte swizzle
    return d;
}
// Tile: 128 rows (tokens) x 256 weight rows.  MODE 1 (gate|up): weight rows
// 0..127 are the gate features f0..f0+127 and rows 128..255 the same up
// features, so one accumulator holds both halves of the SwiGLU; MODE 2 (down):
// weight rows are the outputs d0..d0+255.  The MMA is M = 128 (the rows, A,
// from shared memory by TMA) x N = 256 (the weights, B, dequantised into
// shared memory) x K = 16: at small row counts an instruction costs about the
// same for any N, so the weights take the wide side.
constexpr int kTileRows = 128;             // rows (tokens) per tile: MMA M
constexpr int kTileW = 256;                // weight rows per tile: MMA N
constexpr int kRound = 64;                 // K per round: one 128-byte swizzle atom of fp16
constexpr uint32_t kWRoundBytes = (uint32_t)kTileW * 128;     // a round of the weight operand
constexpr uint32_t kRRoundBytes = (uint32_t)kTileRows * 128;  // a round of the row operand
constexpr int kWBufs = 4;                  // weight rounds in flight: two per dequant half
#ifndef MOE_GEMM_RBUFS
#define MOE_GEMM_RBUFS 3
#endif
#ifndef MOE_GEMM_CSLOTS
#define MOE_GEMM_CSLOTS 3
#endif
constexpr int kRBufs = MOE_GEMM_RBUFS;     // row rounds in flight (they hide the row loads' latency)
// Code stages (2 rounds each: K = 128) in flight.  The weight stream is read
// from HBM by these loads alone, so their depth sets its bandwidth: bytes in
// flight per SM / load latency.
constexpr int kCodeSlots = MOE_GEMM_CSLOTS;
#ifndef MOE_GEMM_CSLOT_BYTES
#define MOE_GEMM_CSLOT_BYTES 16384
#endif
constexpr int kSpr = 2;                    // rounds per code stage: one for each dequant half
constexpr uint32_t kCodeSlotBytes = MOE_GEMM_CSLOT_BYTES;
constexpr int kAccCols = kTileW;           // one accumulator: 128 lanes x 256 fp32 columns
constexpr int kAccBufs = 2;
constexpr uint32_t kGemmSmem = kCodeSlots * kCodeSlotBytes + kWBufs * kWRoundBytes + kRBufs * kRRoundBytes;
static_assert(kAccBufs * kAccCols == 512, "TMEM columns");
static_assert(kGemmSmem + 1024 + 512 <= 232448, "shared memory per block");

// kind::f16, A = B = fp16, D = f32, both K-major, M = 128, N = 256.
MOE_DEVINL uint32_t instr_desc_tile() {
    return (1u << 4) | ((uint32_t)(kTileW >> 3) << 17) | ((uint32_t)(kTileRows >> 4) << 24);
}
// D[tmem] (+)= A[smem] * B[smem]^T; kind::f16 (K = 16) or, with F8, kind::f8f6f4
// (K = 32, both operands e4m3: the format fields of the descriptor are 0 as for fp16)
template <bool F8>
MOE_DEVINL void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
    if constexpr (F8)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
MOE_DEVINL void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
MOE_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
MOE_DEVINL void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
MOE_DEVINL void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Two fp32 values rounded to bf16 (nearest even) and packed: lo in bits 0..15.
MOE_DEVINL uint32_t pack_bf16x2_rn(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// L2 policies: the weight stream is read once (evict first); the activation
// rows are re-read by every weight tile of their group (evict last).
MOE_DEVINL uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
MOE_DEVINL uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
MOE_DEVINL void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
        "%3, %4}], [%5], %6;" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
MOE_DEVINL void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
        "%3}], [%4], %5;" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// Byte offset of the 16-byte chunk c of row r in a K-major 128B-swizzled tile.
MOE_DEVINL uint32_t sw128(int r, int c) { return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)); }

// ---------------------------------------------------------------- grouped GEMM
struct GemmParams {
    const int4* tiles;           // (row0, rows, w0, slot): w0 = first gate feature (MODE 1) / output (MODE 2)
    const int32_t* n_tiles;      // device count
    uint16_t* dst;               // MODE 1: h [rows][F] fp16; MODE 2: y rows [rows][D] bf16
    const uint8_t* scales;       // Q3_S256: the pool's scale base (sub-scales, d)
    size_t stride_s;
    int D, F;
    uint32_t* err;
    uint32_t* dump;              // test hook, normally null: the weight operand of tile dump_tile as the
    int dump_tile;               // MMAs read it, [K / 64 rounds][256 rows][32 f16x2 words]
};

template <int FMT>
struct GemmFmt {
    static constexpr int kCb = FMT == MOE_Q2_32 ? 8 : 12;                  // code bytes per 32 weights
    static constexpr bool kTmaScales = FMT != MOE_Q3_S256;
};

// 16-byte chunk c of row r in a TMA tile of `pitch`-byte rows (32, 64 or 128:
// the swizzle of that width; other pitches are not swizzled).
MOE_DEVINL uint32_t swz_chunk(int r, int c, int pitch) {
    const int sw = (pitch == 32 || pitch == 64 || pitch == 128) ? ((r * pitch) >> 7) & (pitch / 16 - 1) : 0;
    return (uint32_t)(r * pitch + ((c ^ sw) << 4));
}

// One 32-weight block of one weight row -> 16 fp16 pair words: word 8h + i =
// weights (16h + i, 16h + i + 8), each the exact weight rounded once to fp16.
// cw: the block's code words; sm: its (s, m) word (Q2/Q3_32); sc2: sub-scales
// of its two 16-weight halves and d2 (Q3_S256).
template <int FMT>
MOE_DEVINL void dequant_block(const uint32_t (&cw)[3], uint32_t sm, const uint32_t (&sc2)[2], uint32_t d2,
                              const Magic& Mg, uint32_t (&o)[16]) {
    if constexpr (FMT == MOE_Q2_32) {
        const uint32_t s2 = bcast_lo(sm), m2 = bcast_hi(sm);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t w = cw[h], w10 = w >> 10;
            o[8 * h + 0] = w_sm(q2_codes<0>(w, w10, Mg), s2, m2);
            o[8 * h + 1] = w_sm(q2_codes<1>(w, w10, Mg), s2, m2);
            o[8 * h + 2] = w_sm(q2_codes<2>(w, w10, Mg), s2, m2);
            o[8 * h + 3] = w_sm(q2_codes<3>(w, w10, Mg), s2, m2);
            o[8 * h + 4] = w_sm(q2_codes<4>(w, w10, Mg), s2, m2);
            o[8 * h + 5] = w_sm(q2_codes<5>(w, w10, Mg), s2, m2);
            o[8 * h + 6] = w_sm(q2_codes<6>(w, w10, Mg), s2, m2);
            o[8 * h + 7] = w_sm(q2_codes<7>(w, w10, Mg), s2, m2);
        }
    } else {
        const uint32_t s2 = FMT == MOE_Q3_32 ? bcast_lo(sm) : 0u, m2 = FMT == MOE_Q3_32 ? bcast_hi(sm) : 0u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t P, P2;
            q3_group_words(cw[0], cw[1], cw[2], h, P, P2);
            const uint32_t P9 = P >> 9, P10 = P2 >> 10;
            if constexpr (FMT == MOE_Q3_32) {
                o[8 * h + 0] = w_sm(q3_codes<0, false>(P, P9, P2, P10, Mg), s2, m2);
                o[8 * h + 1] = w_sm(q3_codes<1, false>(P, P9, P2, P10, Mg), s2, m2);
                o[8 * h + 2] = w_sm(q3_codes<2, false>(P, P9, P2, P10, Mg), s2, m2);
                o[8 * h + 3] = w_sm(q3_codes<3, false>(P, P9, P2, P10, Mg), s2, m2);
                o[8 * h + 4] = w_sm(q3_codes<4, false>(P, P9, P2, P10, Mg), s2, m2);
                o[8 * h + 5] = w_sm(q3_codes<5, false>(P, P9, P2, P10, Mg), s2, m2);
                o[8 * h + 6] = w_sm(q3_codes<6, false>(P, P9, P2, P10, Mg), s2, m2);
                o[8 * h + 7] = w_sm(q3_codes<7, false>(P, P9, P2, P10, Mg), s2, m2);
            } else {
                o[8 * h + 0] = w_s256(q3_codes<0, true>(P, P9, P2, P10, Mg), sc2[h], d2);
                o[8 * h + 1] = w_s256(q3_codes<1, true>(P, P9, P2, P10, Mg), sc2[h], d2);
                o[8 * h + 2] = w_s256(q3_codes<2, true>(P, P9, P2, P10, Mg), sc2[h], d2);
                o[8 * h + 3] = w_s256(q3_codes<3, true>(P, P9, P2, P10, Mg), sc2[h], d2);
                o[8 * h + 4] = w_s256(q3_codes<4, true>(P, P9, P2, P10, Mg), sc2[h], d2);
                o[8 * h + 5] = w_s256(q3_codes<5, true>(P, P9, P2, P10, Mg), sc2[h], d2);
                o[8 * h + 6] = w_s256(q3_codes<6, true>(P, P9, P2, P10, Mg), sc2[h], d2);
                o[8 * h + 7] = w_s256(q3_codes<7, true>(P, P9, P2, P10, Mg), sc2[h], d2);
            }
        }
    }
}

// Warp roles: 0..15 dequantise (thread i: weight row i % 256, 32-weight block
// i / 256 of each K = 64 round), 16..19 epilogue (TMEM lane quadrant w % 4 =
// rows 32q..), 20 TMA of the code stages (two rounds each), 21 TMA of the row
// operand, 22 MMA issue.  TMEM: two 128 x 256 fp32 accumulators.
template <int FMT, int MODE, bool F8>
__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_scales,
                       const __grid_constant__ CUtensorMap rows128, const __grid_constant__ CUtensorMap rows64,
                       const __grid_constant__ CUtensorMap rows32, const __grid_constant__ CUtensorMap rows16,
                       GemmParams g) {
    using Fm = GemmFmt<FMT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full_c[kCodeSlots], empty_c[kCodeSlots];
    // round b (mod kWBufs): ready = its weights dequantised (one arrive per warp of the
    // half) and its rows landed (the row producer's arrive + bytes); done = its MMAs
    // completed, which frees both its weight buffer and its row buffer
    __shared__ uint64_t ready[kWBufs], done[kWBufs];
    __shared__ uint64_t acc_full[kAccBufs], acc_empty[kAccBufs], drain_bar;
    __shared__ uint32_t tmem_base;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* code_ring = smem;
    uint8_t* w_ring = smem + kCodeSlots * kCodeSlotBytes;
    uint8_t* r_ring = w_ring + kWBufs * kWRoundBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = g.D, F = g.F;
    const int K = MODE == 1 ? D : F;
    // a round is one 128-byte swizzle row of each operand: K = 64 fp16 or K = 128 e4m3
    constexpr int kKR = F8 ? 128 : kRound;
    const int R = K / kKR;                      // rounds per tile
    constexpr int CP = kSpr * 2 * Fm::kCb, SP = kSpr * 8;   // code / scale bytes per weight row of a stage (K = 128)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kCodeSlots; ++s) {
            mbar_init(&full_c[s], 1);
            mbar_init(&empty_c[s], kDqWarps);       // every dequant warp, once it has read the stage
        }
        for (int s = 0; s < kWBufs; ++s) {
            mbar_init(&ready[s], (F8 ? kDqWarps : kDqWarps / 2) + 1);
            mbar_init(&done[s], 1);
        }
        for (int s = 0; s < kAccBufs; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], kEpiWarps); }
        mbar_init(&drain_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    pdl_wait();
    const int n_tiles = __ldg(g.n_tiles);
    __shared__ int dead_s;                      // an earlier kernel gave up: one read for the CTA
    if (threadIdx.x == 0) dead_s = timed_out(g.err) ? 1 : 0;
    __syncthreads();
    const bool dead = dead_s != 0;
    const int first = blockIdx.x, step = gridDim.x;

    if (!dead && warp < kDqWarps) {
        // ---------------- dequantisation into the weight operand (shared memory).  Thread:
        // weight row r and part hp of each code stage (the 16 contiguous code bytes of two
        // 32-weight blocks).  fp16: a round is half a stage; half hp (warps 8hp..8hp+7)
        // takes the rounds of parity hp, i.e. part hp of every stage, and writes the whole
        // 128-byte row of its round into buffer hp or hp + 2 in turn.  e4m3: a round is a
        // stage; all 16 warps take every round, part hp fills bytes [64 hp, 64 hp + 64) of
        // the row, buffers in turn.
        const int r = (int)threadIdx.x & (kTileW - 1), hp = (int)threadIdx.x >> 8;
        constexpr int kStep = F8 ? 1 : 2;          // rounds between two of this thread's rounds
        constexpr int kSeq = F8 ? kWBufs : 2;      // buffers in this thread's sequence
        const Magic Mg = make_magic();
        int li = 0, j = 0;                         // j: this thread's rounds so far
        int cslot = 0;
        uint32_t cph = 0;
        bool ok = true;
        int4 nxt = first < n_tiles ? __ldg(g.tiles + first) : make_int4(0, 0, 0, 0);   // one tile ahead
        for (int tile = first; tile < n_tiles && ok; tile += step, ++li) {
            const int4 td = nxt;
            if (tile + step < n_tiles) nxt = __ldg(g.tiles + tile + step);
            const int w0 = td.z, slot = td.w;
            // Q3_S256: the row's super-block words (sub-scales, d), one super-block ahead of
            // their use so that the loads' latency hides behind the rounds before
            uint32_t sbw[4] = {0, 0, 0, 0}, sbn[4] = {0, 0, 0, 0};
            int sb_cur = -1;
            const uint8_t* sbase = nullptr;
            size_t sb_row = 0, d_row = 0;
            if constexpr (FMT == MOE_Q3_S256) {
                const int pm = MODE == 1 ? (r >> 7) : 2;                   // plane: gate, up, down
                const int wrow = w0 + (MODE == 1 ? (r & 127) : r);
                const size_t blocks = (size_t)D * F / 256;                 // super-blocks per plane
                sbase = g.scales + (size_t)slot * g.stride_s;
                sb_row = (size_t)pm * blocks * 12 + (size_t)wrow * (K / 256) * 12;
                d_row = 3 * blocks * 12 + ((size_t)pm * blocks + (size_t)wrow * (K / 256)) * 2;
                const uint8_t* sp = sbase + sb_row;
                sbn[0] = __ldg(reinterpret_cast<const uint32_t*>(sp));
                sbn[1] = __ldg(reinterpret_cast<const uint32_t*>(sp + 4));
                sbn[2] = __ldg(reinterpret_cast<const uint32_t*>(sp + 8));
                sbn[3] = __ldg(reinterpret_cast<const uint16_t*>(sbase + d_row));
            }
            for (int rr = F8 ? 0 : hp; rr < R; rr += kStep, ++j) {
                if (!mbar_wait_sleep(&full_c[cslot], cph, g.err)) { ok = false; break; }
                const uint8_t* cs = code_ring + cslot * kCodeSlotBytes;
                // both blocks' code bytes [hp * 2 kCb, +2 kCb) and (s, m) words of the row
                uint32_t cw[2][3], sm[2] = {0, 0};
                if constexpr (Fm::kCb == 8) {
                    const uint4 v = *reinterpret_cast<const uint4*>(cs + swz_chunk(r, hp, CP));
                    cw[0][0] = v.x; cw[0][1] = v.y; cw[0][2] = 0;
                    cw[1][0] = v.z; cw[1][1] = v.w; cw[1][2] = 0;
                } else {
                    const uint8_t* rowp = cs + r * CP + hp * 24;              // CP = 48: not swizzled
                    const uint2 a = *reinterpret_cast<const uint2*>(rowp);
                    const uint2 b = *reinterpret_cast<const uint2*>(rowp + 8);
                    const uint2 c = *reinterpret_cast<const uint2*>(rowp + 16);
                    cw[0][0] = a.x; cw[0][1] = a.y; cw[0][2] = b.x;
                    cw[1][0] = b.y; cw[1][1] = c.x; cw[1][2] = c.y;
                }
                if constexpr (Fm::kTmaScales) {
                    const uint2 v = *reinterpret_cast<const uint2*>(cs + kTileW * CP + r * SP + hp * 8);
                    sm[0] = v.x; sm[1] = v.y;
                    if constexpr (F8) {                    // e4m3 operand: weights x 64 (exact in fp16)
                        sm[0] = hmul2u(sm[0], 0x54005400u);
                        sm[1] = hmul2u(sm[1], 0x54005400u);
                    }
                }
                uint32_t sc2[2][2] = {{0, 0}, {0, 0}}, d2 = 0;
                if constexpr (FMT == MOE_Q3_S256) {
                    const int kb0 = F8 ? 4 * rr + 2 * hp : 2 * rr;             // the thread's first block in the row
                    const int sbi = kb0 >> 3;
                    if (sbi != sb_cur) {                   // a new super-block: take the prefetched words
#pragma unroll
                        for (int i = 0; i < 4; ++i) sbw[i] = sbn[i];
                        sb_cur = sbi;
                        if (sbi + 1 < K / 256) {
                            const uint8_t* sp = sbase + sb_row + (size_t)(sbi + 1) * 12;
                            sbn[0] = __ldg(reinterpret_cast<const uint32_t*>(sp));
                            sbn[1] = __ldg(reinterpret_cast<const uint32_t*>(sp + 4));
                            sbn[2] = __ldg(reinterpret_cast<const uint32_t*>(sp + 8));
                            sbn[3] = __ldg(reinterpret_cast<const uint16_t*>(sbase + d_row) + sbi + 1);
                        }
                    }
                    d2 = sbw[3] | (sbw[3] << 16);
                    if constexpr (F8) d2 = hmul2u(d2, 0x54005400u);
                    const uint64_t lo = ((uint64_t)sbw[1] << 32) | sbw[0], hi = ((uint64_t)sbw[2] << 32) | sbw[1];
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int c = (kb0 + b) & 7;                           // sub-blocks 2c, 2c + 1
                        const uint32_t bits = c < 4 ? (uint32_t)(lo >> (12 * c)) : (uint32_t)(hi >> (12 * c - 32));
                        sc2[b][0] = s256_sub(bits & 63u);
                        sc2[b][1] = s256_sub((bits >> 6) & 63u);
                    }
                }
                uint32_t o[2][16];
                dequant_block<FMT>(cw[0], sm[0], sc2[0], d2, Mg, o[0]);
                dequant_block<FMT>(cw[1], sm[1], sc2[1], d2, Mg, o[1]);
                // the stage is released once every value read from it has been used
                const uint32_t dep = o[0][0] ^ o[0][15] ^ o[1][0] ^ o[1][15];
                __syncwarp();
                if (lane == 0) mbar_arrive_dep(&empty_c[cslot], dep);
                if (++cslot == kCodeSlots) { cslot = 0; cph ^= 1u; }
                // the buffer is free once the MMAs of its previous use completed
                const int wb = F8 ? (j & (kWBufs - 1)) : hp + 2 * (j & 1);
                const int use = j / kSeq;
                if (use >= 1) {
                    if (!mbar_wait_sleep(&done[wb], (use - 1) & 1, g.err)) { ok = false; break; }
                    tc_fence_after();
                }
                uint8_t* wbuf = w_ring + wb * kWRoundBytes;
                if constexpr (F8) {
                    // e4m3 pairs: word i of a block's fp16 pairs (16h + i, 16h + i + 8) -> bytes 2i, 2i + 1
#pragma unroll
                    for (int b = 0; b < 2; ++b)
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            uint32_t e[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                e[i] = e4m3x2_of_f16x2(o[b][8 * q + 2 * i]) | (e4m3x2_of_f16x2(o[b][8 * q + 2 * i + 1]) << 16);
                            *reinterpret_cast<uint4*>(wbuf + sw128(r, 4 * hp + 2 * b + q)) = make_uint4(e[0], e[1], e[2], e[3]);
                        }
                } else {
#pragma unroll
                    for (int b = 0; b < 2; ++b)
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<uint4*>(wbuf + sw128(r, 4 * b + q)) =
                                make_uint4(o[b][4 * q], o[b][4 * q + 1], o[b][4 * q + 2], o[b][4 * q + 3]);
                    if (g.dump != nullptr && tile == g.dump_tile) {
                        // test hook: the round's weight operand as the MMAs will read it
                        uint32_t* drow = g.dump + ((size_t)rr * kTileW + r) * 32;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 v = *reinterpret_cast<const uint4*>(wbuf + sw128(r, q));
                            drow[4 * q] = v.x; drow[4 * q + 1] = v.y; drow[4 * q + 2] = v.z; drow[4 * q + 3] = v.w;
                        }
                    }
                }
                fence_proxy_async();                 // generic stores -> the tensor core's reads
                __syncwarp();
                if (lane == 0) mbar_arrive(&ready[wb]);
            }
        }
    } else if (!dead && warp < kTmaWarp) {
        // ---------------- epilogue: TMEM -> registers -> global; lane = row of the tile
        constexpr float kDescale = F8 ? 0.015625f : 1.0f;    // e4m3 weights carry a factor 64
        const int q = warp & 3;
        const int t = 32 * q + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
        int li = 0;
        bool range_bad = false;
        int4 nxt = first < n_tiles ? __ldg(g.tiles + first) : make_int4(0, 0, 0, 0);   // one tile ahead
        for (int tile = first; tile < n_tiles; tile += step, ++li) {
            const int4 td = nxt;
            if (tile + step < n_tiles) nxt = __ldg(g.tiles + tile + step);
            const int row0 = td.x, nrows = td.y, w0 = td.z;
            const int ab = li & 1;
            if (!mbar_wait_sleep(&acc_full[ab], (li >> 1) & 1, g.err)) break;
            tc_fence_after();
            const uint32_t acc = lane_addr + (uint32_t)(ab * kAccCols);
            if constexpr (MODE == 1) {
                // columns c: gate feature w0 + c, columns 128 + c: the same up feature
                for (int c = 0; c < kTileW / 2; c += 16) {
                    uint32_t gv[16], uv[16];
                    tmem_ld16(acc + (uint32_t)c, gv);
                    tmem_ld16(acc + (uint32_t)(kTileW / 2 + c), uv);
                    tmem_ld_wait();
                    if (F8 && t < nrows) {
                        // acc = 64 x the products (the e4m3 weights carry a factor 64); h in e4m3, the 16
                        // features in the K order of the down GEMM's row operand: bytes 2i, 2i + 1 = (i, i + 8)
                        uint32_t e[4] = {0, 0, 0, 0};
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float g0 = __uint_as_float(gv[i]) * kDescale, u0 = __uint_as_float(uv[i]) * kDescale;
                            const float g1 = __uint_as_float(gv[i + 8]) * kDescale, u1 = __uint_as_float(uv[i + 8]) * kDescale;
                            const float h0 = g0 / (1.0f + expf(-g0)) * u0, h1 = g1 / (1.0f + expf(-g1)) * u1;
                            range_bad |= !(fabsf(h0) < 448.f) || !(fabsf(h1) < 448.f);
                            e[i >> 1] |= e4m3x2_of_f32(h0, h1) << (16 * (i & 1));
                        }
                        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(g.dst) + (size_t)(row0 + t) * F + w0 + c) =
                            make_uint4(e[0], e[1], e[2], e[3]);
                    } else if (t < nrows) {
                        // the 16 features in the K order of the down GEMM's row operand: word i = (i, i + 8);
                        // h is a bf16 value, carried exactly in fp16 when in range
                        uint32_t w[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float g0 = __uint_as_float(gv[i]), u0 = __uint_as_float(uv[i]);
                            const float g1 = __uint_as_float(gv[i + 8]), u1 = __uint_as_float(uv[i + 8]);
                            const uint32_t hp = pack_bf16x2_rn(g0 / (1.0f + expf(-g0)) * u0, g1 / (1.0f + expf(-g1)) * u1);
                            const float h0 = __uint_as_float(hp << 16), h1 = __uint_as_float(hp & 0xffff0000u);
                            range_bad |= !(fabsf(h0) < 65520.f) || !(fabsf(h1) < 65520.f);
                            const __half2 hh = __floats2half2_rn(h0, h1);
                            w[i] = *reinterpret_cast<const uint32_t*>(&hh);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(g.dst + (size_t)(row0 + t) * F + w0 + c);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            } else {
                if (32 * q < nrows) {                    // a quadrant with no rows of the tile skips its loads
                    for (int c = 0; c < kTileW; c += 32) {   // two loads in flight per wait
                        uint32_t v[2][16];
                        tmem_ld16(acc + (uint32_t)c, v[0]);
                        tmem_ld16(acc + (uint32_t)(c + 16), v[1]);
                        tmem_ld_wait();
                        if (t < nrows) {
                            uint4* dst = reinterpret_cast<uint4*>(g.dst + (size_t)(row0 + t) * D + w0 + c);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                uint32_t w[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    w[i] = pack_bf16x2_rn(__uint_as_float(v[h][2 * i]) * kDescale,
                                                          __uint_as_float(v[h][2 * i + 1]) * kDescale);
                                dst[2 * h] = make_uint4(w[0], w[1], w[2], w[3]);
                                dst[2 * h + 1] = make_uint4(w[4], w[5], w[6], w[7]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
        if (range_bad) atomicOr(g.err, kErrRange);
    } else if (!dead && warp == kTmaWarp) {
        // ---------------- TMA loads of the code (and scale) stages: rows 0..127 and 128..255
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            const uint32_t bytes = (uint32_t)kTileW * CP + (Fm::kTmaScales ? (uint32_t)kTileW * SP : 0u);
            int issued = 0, cst = 0, slot = 0;
            uint32_t ph = 0;
            bool ok = true;
            int4 nxt = first < n_tiles ? __ldg(g.tiles + first) : make_int4(0, 0, 0, 0);   // one tile ahead
            for (int tile = first; tile < n_tiles && ok; tile += step) {
                const int4 td = nxt;
                if (tile + step < n_tiles) nxt = __ldg(g.tiles + tile + step);
                const int w0 = td.z, slot_id = td.w;
                for (int c = 0; c < K / 128; ++c, ++cst) {
                    if (cst >= kCodeSlots && !mbar_wait_sleep(&empty_c[slot], ph ^ 1u, g.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* cs = code_ring + slot * kCodeSlotBytes;
                    mbar_arrive_expect_tx(&full_c[slot], bytes);
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        // MODE 1: gate rows w0.., then up rows F + w0..; MODE 2: outputs w0.., w0 + 128..
                        const int y = MODE == 1 ? m * F + w0 : w0 + 128 * m;
                        tma_load_3d(smem_u32(cs + m * 128 * CP), &map_codes, c * CP, y, slot_id, &full_c[slot], pol);
                        if constexpr (Fm::kTmaScales)
                            tma_load_3d(smem_u32(cs + kTileW * CP + m * 128 * SP), &map_scales, c * SP, y, slot_id,
                                        &full_c[slot], pol);
                    }
                    issued = cst + 1;
                    if (++slot == kCodeSlots) { slot = 0; ph ^= 1u; }
                }
            }
            // every issued stage completes before the CTA exits
            for (int j = issued - kCodeSlots; j < issued; ++j)
                if (j >= 0) mbar_drain(&full_c[j % kCodeSlots], (j / kCodeSlots) & 1);
        }
        __syncwarp();
    } else if (!dead && warp == kGatherWarp) {
        // ---------------- row operand: the tile's rows x 64 K per round (K-major, 128B
        // swizzle) in one box of 16, 32, 64 or 128 rows; the rest of the round's
        // 128 MMA rows hold stale values, whose results are not stored
        if (lane == 0) {
            const uint64_t pol = l2_evict_last();
            bool ok = true;
            int issued = 0, gr = 0, rb = 0, b = 0, lb = 0;      // lb: round gr - kRBufs (mod kWBufs)
            uint32_t ph = 0, lph = 0;
            int4 nxt = first < n_tiles ? __ldg(g.tiles + first) : make_int4(0, 0, 0, 0);   // one tile ahead
            for (int tile = first; tile < n_tiles && ok; tile += step) {
                const int4 td = nxt;
                if (tile + step < n_tiles) nxt = __ldg(g.tiles + tile + step);
                const int row0 = td.x, nrows = td.y;
                const CUtensorMap* m = nrows > 64 ? &rows128 : nrows > 32 ? &rows64 : nrows > 16 ? &rows32 : &rows16;
                const uint32_t bytes = (nrows > 64 ? 128u : nrows > 32 ? 64u : nrows > 16 ? 32u : 16u) * 128u;
                for (int rr = 0; rr < R; ++rr, ++gr) {
                    if (gr >= kRBufs) {      // row buffer rb is free once round gr - kRBufs is done
                        if (!mbar_wait_sleep(&done[lb], lph, g.err)) { ok = false; break; }
                        if (++lb == kWBufs) { lb = 0; lph ^= 1u; }
                    }
                    mbar_arrive_expect_tx(&ready[b], bytes);
                    tma_load_2d(smem_u32(r_ring + rb * kRRoundBytes), m, rr * kKR, row0, &ready[b], pol);
                    issued = gr + 1;
                    if (++rb == kRBufs) rb = 0;
                    if (++b == kWBufs) { b = 0; ph ^= 1u; }
                }
            }
            // every issued row load lands before the CTA exits
            for (int j = issued - kRBufs; j < issued; ++j)
                if (j >= 0) mbar_drain(&ready[j % kWBufs], (j / kWBufs) & 1);
        }
        __syncwarp();
    } else if (!dead && warp == kMmaWarp) {
        // ---------------- single-thread MMA issue: per round, 4 MMAs of K = 16
        if (lane == 0) {
            const uint32_t idesc = instr_desc_tile();
            int li = 0, wb = 0, rb = 0;
            uint32_t wph = 0;
            bool ok = true, issued = false;
            bool pre = false;                            // the round's ready phase already seen complete
            for (int tile = first; tile < n_tiles && ok; tile += step, ++li) {
                const int ab = li & 1;
                if (li >= kAccBufs) {
                    if (!mbar_wait_sleep(&acc_empty[ab], ((li >> 1) - 1) & 1, g.err)) { ok = false; break; }
                    tc_fence_after();
                }
                const uint32_t d_tmem = tmem + (uint32_t)(ab * kAccCols);
                for (int rr = 0; rr < R; ++rr) {
                    if (!pre && !mbar_wait_sleep(&ready[wb], wph, g.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(smem_u32(r_ring + rb * kRRoundBytes));
                    const uint64_t bd = smem_desc_sw128(smem_u32(w_ring + wb * kWRoundBytes));
                    // test the next round's barrier now: the test's latency then passes while
                    // this round's MMAs hold the thread (a phase, once complete, stays so until
                    // the round's MMAs are done)
                    const int nb = wb + 1 == kWBufs ? 0 : wb + 1;
                    const uint32_t nph = wb + 1 == kWBufs ? wph ^ 1u : wph;
                    pre = mbar_try_wait(&ready[nb], nph);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)     // 32 bytes of K per MMA: descriptor start in 16-byte units
                        mma_ss<F8>(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (rr > 0 || kk > 0) ? 1u : 0u);
                    issued = true;
                    mma_commit(&done[wb]);               // frees the round's weight and row buffers
                    wb = nb;
                    wph = nph;
                    if (++rb == kRBufs) rb = 0;
                }
                if (ok) mma_commit(&acc_full[ab]);
            }
            if (issued) {                                // every MMA completes before TMEM is released
                mma_commit(&drain_bar);
                mbar_drain(&drain_bar, 0);
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

// ---------------------------------------------------------------- host: tensor maps and launches
// A byte tensor [slots][rows][row_bytes] (slot stride given), boxes of
// box_x bytes x box_y rows.
bool byte_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t slots,
              uint64_t slot_stride, uint32_t box_x, uint32_t box_y, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {row_bytes, rows, slots};
    const cuuint64_t strides[2] = {row_bytes, slot_stride};
    const cuuint32_t box[3] = {box_x, box_y, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The row operand: fp16 [rows][K] with boxes of 64 x box_rows, or e4m3 bytes
// [rows][K] with boxes of 128 x box_rows (F8); 128B swizzle.
bool row_map(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows, bool f8) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * (f8 ? 1 : 2)};
    const cuuint32_t box[2] = {(cuuint32_t)(f8 ? 128 : kRound), box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims,
              strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for(uint32_t pitch) {
    return pitch == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                        : pitch == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : pitch == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE;
}

template <int FMT, int MODE, bool F8>
moe_status launch_gemm(const PoolView& P, GemmParams prm, const void* src, uint64_t src_rows, int max_tiles,
                       cudaStream_t s) {
    using Fm = GemmFmt<FMT>;
    const int D = P.D, F = P.F;
    const int Kg = MODE == 1 ? D : F;                 // K of the matrix set
    const uint64_t rows = MODE == 1 ? 2 * (uint64_t)F : (uint64_t)D;
    const uint64_t code_row = (uint64_t)Kg / 32 * Fm::kCb;
    const uint8_t* codes = P.codes + (MODE == 1 ? 0 : 2 * (uint64_t)F * ((uint64_t)D / 32 * Fm::kCb));
    CUtensorMap mc, ms, mr;
    const uint32_t cp = (uint32_t)(kSpr * 2 * Fm::kCb), sp = (uint32_t)(kSpr * 8);
    if ((uint64_t)kTileW * (cp + (Fm::kTmaScales ? sp : 0u)) > kCodeSlotBytes || Kg % 128) return MOE_ERR_UNSUPPORTED;
    // code (and scale) stages: two boxes of 128 weight rows
    if (!byte_map(&mc, codes, code_row, rows, (uint64_t)P.n_slots, P.stride_c, cp, 128, swizzle_for(cp)))
        return MOE_ERR_CUDA;
    if constexpr (Fm::kTmaScales) {
        const uint64_t scale_row = (uint64_t)Kg / 32 * 4;
        const uint8_t* scales = P.scales + (MODE == 1 ? 0 : 2 * (uint64_t)F * ((uint64_t)D / 32 * 4));
        if (!byte_map(&ms, scales, scale_row, rows, (uint64_t)P.n_slots, P.stride_s, sp, 128, swizzle_for(sp)))
            return MOE_ERR_CUDA;
    } else {
        ms = mc;
    }
    CUtensorMap r64, r32, r16;
    if (!row_map(&mr, src, (uint64_t)Kg, src_rows, 128, F8) || !row_map(&r64, src, (uint64_t)Kg, src_rows, 64, F8) ||
        !row_map(&r32, src, (uint64_t)Kg, src_rows, 32, F8) || !row_map(&r16, src, (uint64_t)Kg, src_rows, 16, F8))
        return MOE_ERR_CUDA;
    const size_t smem = kGemmSmem + 1024;
    static std::atomic<uint64_t> attr{0};
    if (!once_per_device(attr, [&] {
            return cudaFuncSetAttribute(expert_gemm_kernel<FMT, MODE, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem) == cudaSuccess;
        }))
        return MOE_ERR_CUDA;
    const int grid = max_tiles < device_sm_count() ? (max_tiles > 0 ? max_tiles : 1) : device_sm_count();
    const cudaError_t e = launch_pdl(expert_gemm_kernel<FMT, MODE, F8>, dim3(grid), dim3(kGemmThreads), smem, s, mc, ms,
                                     mr, r64, r32, r16, prm);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int FMT, bool F8>
moe_status launch_gemms(const PoolView& P, const PrefillWs& w, uint16_t* yrows, const WsSizes& sz, int T, int k,
                        cudaStream_t s) {
    GemmParams a1;
    a1.tiles = w.tiles1; a1.n_tiles = w.meta + 1; a1.dst = w.h;
    a1.scales = P.scales; a1.stride_s = P.stride_s; a1.D = P.D; a1.F = P.F; a1.err = w.err;
    a1.dump = nullptr; a1.dump_tile = -1;
    const uint64_t rows = (uint64_t)T * (k + 1);
    moe_status st = launch_gemm<FMT, 1, F8>(P, a1, w.xg, rows, (int)sz.max_t1, s);
    if (st != MOE_OK) return st;
    GemmParams a2 = a1;
    a2.tiles = w.tiles2; a2.n_tiles = w.meta + 2; a2.dst = yrows;
    return launch_gemm<FMT, 2, F8>(P, a2, w.h, rows, (int)sz.max_t2, s);
}

template <int FMT>
moe_status launch_operand_dump(const PoolView& P, int gemm, int slot, int m0, uint32_t* dump, void* ws, cudaStream_t s) {
    // ws: [0, 1024) error word + tile list + count, then a zero row operand of
    // 128 rows x max(D, F) fp16 (every row box of the tensor maps fits), then 16
    // rows of output
    char* p = reinterpret_cast<char*>(ws);
    const int Kmax = P.D > P.F ? P.D : P.F;
    uint16_t* src = reinterpret_cast<uint16_t*>(p + 1024);
    uint16_t* dst = reinterpret_cast<uint16_t*>(p + 1024 + (size_t)128 * Kmax * 2);
    int4* tiles = reinterpret_cast<int4*>(p + 256);
    int32_t* count = reinterpret_cast<int32_t*>(p + 512);
    const int4 td = make_int4(0, 16, m0, slot);
    const int32_t one = 1;
    if (cudaMemsetAsync(p, 0, 1024 + (size_t)128 * Kmax * 2, s) != cudaSuccess ||
        cudaMemcpyAsync(tiles, &td, sizeof(td), cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(count, &one, sizeof(one), cudaMemcpyHostToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    GemmParams a;
    a.tiles = tiles; a.n_tiles = count; a.dst = dst;
    a.scales = P.scales; a.stride_s = P.stride_s; a.D = P.D; a.F = P.F;
    a.err = reinterpret_cast<uint32_t*>(p + 4);
    a.dump = dump; a.dump_tile = 0;
    return gemm == 1 ? launch_gemm<FMT, 1, false>(P, a, src, 128, 1, s) : launch_gemm<FMT, 2, false>(P, a, src, 128, 1, s);
}

}  // namespace

size_t prefill_operand_dump_ws_bytes(int D, int F) { return 1024 + (size_t)144 * (D > F ? D : F) * 2; }

moe_status launch_prefill_operand_dump(const PoolView& P, int gemm, int slot, int m0, uint32_t* dump, void* ws,
                                       cudaStream_t s) {
    if (P.F % kKAlign || P.D % kKAlign || P.D % kDownRows) return MOE_ERR_UNSUPPORTED;
    if (!encode_tiled()) return MOE_ERR_CUDA;
    switch (P.fmt) {
        case MOE_Q2_32: return launch_operand_dump<MOE_Q2_32>(P, gemm, slot, m0, dump, ws, s);
        case MOE_Q3_32: return launch_operand_dump<MOE_Q3_32>(P, gemm, slot, m0, dump, ws, s);
        default: return launch_operand_dump<MOE_Q3_S256>(P, gemm, slot, m0, dump, ws, s);
    }
}

size_t prefill_workspace_bytes(int T, int D, int F, int E, int k) { return ws_sizes(T, D, F, E, k).total; }

moe_status launch_prefill_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x, int T,
                                  const int32_t* ids, int k, void* expert_out, int32_t* miss_list,
                                  int32_t* miss_count, void* ws, cudaStream_t s, bool fp8) {
    if (P.F % kKAlign || P.D % kDownRows || E > kMaxE) return MOE_ERR_UNSUPPORTED;
    if (!encode_tiled()) return MOE_ERR_CUDA;
    const PrefillWs w = carve(ws, T, P.D, P.F, E, k);
    PlanArgs a;
    a.ids = ids; a.slot_table = slot_table; a.T = T; a.k = k; a.E = E; a.n_slots = P.n_slots;
    a.shared_slot = P.shared_slot; a.F = P.F; a.D = P.D; a.w = w;
    a.rowmap = reinterpret_cast<int32_t*>(expert_out);
    a.miss_list = miss_list;
    a.miss_count = miss_count;
    const int nchunk = (T + kChunk - 1) / kChunk;
    cudaError_t e = launch_pdl(plan_count_kernel, dim3(nchunk), dim3(kChunk), 0, s, a);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_pdl(plan_scan_kernel, dim3(1), dim3(1024), 0, s, a);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_pdl(plan_scatter_kernel, dim3(nchunk), dim3(kChunk), 0, s, a);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const dim3 ggrid((unsigned)((size_t)T * (k + 1)));     // rows: at most T k routed + T shared
    e = fp8 ? launch_pdl(gather_f8p_kernel, ggrid, dim3(kGatherThreads), 0, s, x, w.perm, w.meta, T, P.D,
                         reinterpret_cast<uint8_t*>(w.xg), w.err)
            : launch_pdl(gather_f16p_kernel, ggrid, dim3(kGatherThreads), 0, s, x, w.perm, w.meta, T, P.D, w.xg, w.err);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const WsSizes sz = ws_sizes(T, P.D, P.F, E, k);
    uint16_t* yrows = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(expert_out) + rowmap_bytes(T, k));
    if (fp8) {
        switch (P.fmt) {
            case MOE_Q2_32: return launch_gemms<MOE_Q2_32, true>(P, w, yrows, sz, T, k, s);
            case MOE_Q3_32: return launch_gemms<MOE_Q3_32, true>(P, w, yrows, sz, T, k, s);
            default: return launch_gemms<MOE_Q3_S256, true>(P, w, yrows, sz, T, k, s);
        }
    }
    switch (P.fmt) {
        case MOE_Q2_32: return launch_gemms<MOE_Q2_32, false>(P, w, yrows, sz, T, k, s);
        case MOE_Q3_32: return launch_gemms<MOE_Q3_32, false>(P, w, yrows, sz, T, k, s);
        default: return launch_gemms<MOE_Q3_S256, false>(P, w, yrows, sz, T, k, s);
    }
}

}  // namespace moe
