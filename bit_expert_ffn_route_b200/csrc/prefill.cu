// prefill.cu — expert pass for chunks of many tokens (T > 4): a deterministic
// tokens-by-expert permute, then two grouped GEMMs on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory) whose weight operand is
// dequantised from the 2-/3-bit blocks into shared memory on the fly.
//
// The pages: prefill runs in chunks, with expert transfers overlapped with GPU
// compute (greenbean-ai "Strata 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next" §三);
// 10 routed + 1 shared experts per token (wiselychen RTX 5090 report,
// "30 秒定位"); weights are 2-3.5 bit block-quantised (wiselychen report §1).
//
// Rows.  Every resident (token, rank) pair and every token's shared-expert
// evaluation is one row; rows are grouped by expert (routed experts in id
// order, tokens ascending within an expert), then the T shared rows.
//   GEMM 1 (gate|up): per tile of 128 features x up to 256 rows of one group,
//     acc_g = Wg x, acc_u = Wu x in TMEM; epilogue h = bf16(silu(acc_g) * acc_u)
//   GEMM 2 (down): per tile of 128 outputs x up to 256 rows, acc = Wd h;
//     epilogue y = bf16(acc) into the expert_out rows
// Both are "swap-AB": the weights are the M = 128 operand, the rows are N.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

namespace moe {
namespace {

constexpr int kChunk = 256;            // tokens per plan chunk
constexpr int kMaxE = 1024;
constexpr int kTileM = 128;
constexpr int kTileN = 256;            // max rows per tile
constexpr int kTileK = 64;             // one 128-byte swizzle atom of bf16
constexpr int kStages = 3;
constexpr int kDqWarps = 8;            // dequant + epilogue warps
constexpr int kThreads = (kDqWarps + 2) * 32;   // + B gather warp + MMA warp
constexpr int kGatherWarp = kDqWarps;
constexpr int kMmaWarp = kDqWarps + 1;

// ---------------------------------------------------------------- workspace
struct PrefillWs {
    int32_t* hist;        // [nchunk][E]: hits of expert e in the chunk, then the chunk's base row
    int32_t* miss_hist;   // [nchunk]: misses in the chunk, then the chunk's base index
    int32_t* meta;        // [0] rows of routed groups, [1] tiles1, [2] tiles2
    int4* tiles1;         // (group row0, rows, m0, slot)
    int4* tiles2;
    int32_t* perm;        // [rows] token of each row
    uint16_t* h;          // [rows][F] bf16
    uint32_t* err;
};

inline size_t align256(size_t n) { return (n + 255) / 256 * 256; }

struct WsSizes {
    size_t hist, miss, meta, t1, t2, perm, h, total;
};

inline WsSizes ws_sizes(int T, int D, int F, int E, int k) {
    const int nchunk = (T + kChunk - 1) / kChunk;
    const size_t rows = (size_t)T * (k + 1);
    const size_t ntiles = rows / kTileN + (size_t)E + 2;   // bound on sum over groups of ceil(n/256)
    WsSizes s;
    s.hist = align256((size_t)nchunk * E * 4);
    s.miss = align256((size_t)nchunk * 4);
    s.meta = 256;
    s.t1 = align256(ntiles * (F / kTileM) * sizeof(int4));
    s.t2 = align256(ntiles * (D / kTileM) * sizeof(int4));
    s.perm = align256(rows * 4);
    s.h = align256(rows * F * 2);
    s.total = 1024 + s.hist + s.miss + s.meta + s.t1 + s.t2 + s.perm + s.h;
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
__device__ void chunk_masks(const PlanArgs& a, int chunk, uint32_t (*mask)[kChunk / 32], int& my_miss) {
    for (int i = threadIdx.x; i < a.E * (kChunk / 32); i += blockDim.x) mask[i / (kChunk / 32)][i % (kChunk / 32)] = 0;
    __syncthreads();
    const int t = chunk * kChunk + threadIdx.x;
    my_miss = 0;
    if (t < a.T) {
        for (int r = 0; r < a.k; ++r) {
            const int e = __ldg(a.ids + (size_t)t * a.k + r);
            if (plan_slot(a, e) >= 0) atomicOr(&mask[e][threadIdx.x >> 5], 1u << (threadIdx.x & 31));
            else ++my_miss;
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kChunk) plan_count_kernel(PlanArgs a) {
    __shared__ uint32_t mask[kMaxE][kChunk / 32];
    __shared__ int wsum[kChunk / 32];
    pdl_wait();
    int my_miss;
    chunk_masks(a, blockIdx.x, mask, my_miss);
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
__global__ void __launch_bounds__(1024) plan_scan_kernel(PlanArgs a) {
    __shared__ int tot[kMaxE];
    __shared__ int off[kMaxE + 1];
    __shared__ int t1off[kMaxE + 2];
    pdl_wait();
    const int nchunk = (a.T + kChunk - 1) / kChunk;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = 0;
        for (int c = 0; c < nchunk; ++c) run += a.w.hist[(size_t)c * a.E + e];
        tot[e] = run;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < a.E; ++e) { off[e] = run; run += tot[e]; }
        off[a.E] = run;
        // misses: exclusive scan over chunks (token-major order)
        int m = 0;
        for (int c = 0; c < nchunk; ++c) { const int v = a.w.miss_hist[c]; a.w.miss_hist[c] = m; m += v; }
        a.miss_count[0] = m;
        a.w.meta[0] = run;
        // tile counts per group (routed groups in id order, then the shared group)
        int nt = 0;
        for (int e = 0; e <= a.E; ++e) {
            t1off[e] = nt;
            const int n = e < a.E ? tot[e] : a.T;
            nt += (n + kTileN - 1) / kTileN;
        }
        t1off[a.E + 1] = nt;
        a.w.meta[1] = nt * (a.F / kTileM);
        a.w.meta[2] = nt * (a.D / kTileM);
    }
    __syncthreads();
    // per-chunk base rows of every expert
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = off[e];
        for (int c = 0; c < nchunk; ++c) {
            const int v = a.w.hist[(size_t)c * a.E + e];
            a.w.hist[(size_t)c * a.E + e] = run;
            run += v;
        }
    }
    // tile lists: group e (or the shared group), n-tile, m-tile
    const int mt1 = a.F / kTileM, mt2 = a.D / kTileM;
    for (int g = threadIdx.x; g <= a.E; g += blockDim.x) {
        const int n = g < a.E ? tot[g] : a.T;
        const int row0 = g < a.E ? off[g] : off[a.E];
        const int slot = g < a.E ? (n > 0 ? plan_slot(a, g) : -1) : a.shared_slot;
        const int first = t1off[g], cnt = t1off[g + 1] - first;
        for (int j = 0; j < cnt; ++j) {
            const int r0 = row0 + j * kTileN, rows = min(kTileN, n - j * kTileN);
            for (int m = 0; m < mt1; ++m) a.w.tiles1[(size_t)(first + j) * mt1 + m] = make_int4(r0, rows, m * kTileM, slot);
            for (int m = 0; m < mt2; ++m) a.w.tiles2[(size_t)(first + j) * mt2 + m] = make_int4(r0, rows, m * kTileM, slot);
        }
    }
}

// Rows of every hit (stable: tokens ascending within an expert), the row map,
// the shared rows and the miss list (token-major, rank order).
__global__ void __launch_bounds__(kChunk) plan_scatter_kernel(PlanArgs a) {
    __shared__ uint32_t mask[kMaxE][kChunk / 32];
    __shared__ int wsum[kChunk / 32];
    pdl_wait();
    int my_miss;
    chunk_masks(a, blockIdx.x, mask, my_miss);
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
    for (int r = 0; r < k; ++r) {
        const int e = __ldg(a.ids + (size_t)t * k + r);
        if (plan_slot(a, e) >= 0) {
            int below = 0;
            const int wi = threadIdx.x >> 5;
            for (int w = 0; w < wi; ++w) below += __popc(mask[e][w]);
            below += __popc(mask[e][wi] & ((1u << (threadIdx.x & 31)) - 1u));
            const int row = a.w.hist[(size_t)blockIdx.x * a.E + e] + below;
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

// ---------------------------------------------------------------- tcgen05 helpers
MOE_DEVINL uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3ffffu) >> 4);        // start address
    d |= (uint64_t)1 << 16;                           // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024 >> 4) << 32;                 // stride byte offset: 8-row groups
    d |= (uint64_t)1 << 46;                           // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                           // 128-byte swizzle
    return d;
}
// kind::f16, A = B = bf16, D = f32, both K-major, M = 128.
MOE_DEVINL uint32_t instr_desc(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTileM >> 4) << 24);
}
MOE_DEVINL void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
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
MOE_DEVINL void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
MOE_DEVINL void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
MOE_DEVINL void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Byte offset of the 16-byte chunk c of row r in a K-major 128B-swizzled tile.
MOE_DEVINL uint32_t sw128(int r, int c) { return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)); }

MOE_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------- dequantisation
// Exact weights w = fmaf(s, q, m) (Q2_32 / Q3_32) or d (sc - 32)(q - 4)
// (Q3_S256) for 32 consecutive codes, then rounded to bf16 (nearest even).
// Codes are taken from their words with the same bit-field logic as the
// format definition: bit stream position nbits * j.
template <int NB>
MOE_DEVINL int field(const uint32_t* w, int j) {
    const int bit = NB * j, wi = bit >> 5, sh = bit & 31;
    const uint32_t lo = w[wi];
    const uint32_t hi = (sh + NB > 32) ? w[wi + 1] : 0u;
    return (int)(__funnelshift_r(lo, hi, sh) & ((1u << NB) - 1u));
}

template <int FMT>
struct Dq {
    static constexpr int kCodeChunk = (FMT == MOE_Q2_32) ? 8 : 12;   // code bytes per 32 weights
    static constexpr int kBlock = (FMT == MOE_Q3_S256) ? 256 : 32;
    static constexpr int kBlockCode = (FMT == MOE_Q2_32) ? 8 : (FMT == MOE_Q3_32 ? 12 : 96);
};

// Dequantise 32 weights (chunk cb of row `row`, K weights per row) of plane pl
// into 16 packed bf16 pairs.
template <int FMT>
MOE_DEVINL void dequant32(const uint8_t* cplane, const uint8_t* mplane, const uint8_t* dplane, int row, int K, int cb,
                          uint32_t (&out)[16]) {
    uint32_t w[3];
    float wv[32];
    if constexpr (FMT == MOE_Q3_S256) {
        const int nsb = K / 256, sb = cb >> 3, j = cb & 7;
        const size_t blk = (size_t)row * nsb + sb;
        const uint8_t* p = cplane + blk * 96 + j * 12;
        w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
        w[1] = __ldg(reinterpret_cast<const uint32_t*>(p + 4));
        w[2] = __ldg(reinterpret_cast<const uint32_t*>(p + 8));
        const uint32_t* scp = reinterpret_cast<const uint32_t*>(mplane + blk * 12);
        uint32_t sw[3] = {__ldg(scp), __ldg(scp + 1), __ldg(scp + 2)};
        const float d = f16_bits_to_f32(__ldg(reinterpret_cast<const uint16_t*>(dplane) + blk));
        const int s0 = field<6>(sw, 2 * j), s1 = field<6>(sw, 2 * j + 1);
        const float S0 = d * (float)(s0 - 32), S1 = d * (float)(s1 - 32);   // exact
#pragma unroll
        for (int i = 0; i < 32; ++i) wv[i] = (i < 16 ? S0 : S1) * (float)(field<3>(w, i) - 4);   // exact
    } else {
        const size_t blk = (size_t)row * (K / 32) + cb;
        const uint8_t* p = cplane + blk * Dq<FMT>::kCodeChunk;
        if constexpr (FMT == MOE_Q2_32) {
            const uint2 c = __ldg(reinterpret_cast<const uint2*>(p));
            w[0] = c.x; w[1] = c.y; w[2] = 0;
        } else {
            w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
            w[1] = __ldg(reinterpret_cast<const uint32_t*>(p + 4));
            w[2] = __ldg(reinterpret_cast<const uint32_t*>(p + 8));
        }
        const float2 sm = __half22float2(*reinterpret_cast<const __half2*>(mplane + blk * 4));
        constexpr int NB = (FMT == MOE_Q2_32) ? 2 : 3;
#pragma unroll
        for (int i = 0; i < 32; ++i) wv[i] = __fmaf_rn(sm.x, (float)field<NB>(w, i), sm.y);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) out[i] = pack_bf16x2(wv[2 * i], wv[2 * i + 1]);
}

template <int FMT>
struct PlanesP {
    const uint8_t* c;
    const uint8_t* m;
    const uint8_t* d;
};
template <int FMT>
MOE_DEVINL PlanesP<FMT> pplanes(const PoolView& P, int slot, int mat) {
    const size_t blocks = (size_t)P.D * P.F / Dq<FMT>::kBlock;
    PlanesP<FMT> pl;
    pl.c = P.codes + (size_t)slot * P.stride_c + (size_t)mat * blocks * Dq<FMT>::kBlockCode;
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

// ---------------------------------------------------------------- grouped GEMM
struct GemmArgs {
    PoolView P;
    const int4* tiles;
    const int32_t* n_tiles;      // device count
    const uint16_t* src;         // MODE 1: x [T][D]; MODE 2: h [rows][F]
    const int32_t* perm;         // MODE 1: token of each row
    uint16_t* dst;               // MODE 1: h [rows][F]; MODE 2: y rows [rows][D]
    uint32_t* err;
};

// MODE 1: gate|up (two accumulators, K = D, SwiGLU epilogue into h).
// MODE 2: down (one accumulator, K = F, epilogue into the y rows).
template <int FMT, int MODE>
__global__ void __launch_bounds__(kThreads, 1) expert_gemm_kernel(GemmArgs g) {
    constexpr int NMAT = (MODE == 1) ? 2 : 1;
    constexpr uint32_t kA = kTileM * kTileK * 2;            // 16 KB per weight matrix
    constexpr uint32_t kB = kTileN * kTileK * 2;            // 32 KB
    constexpr uint32_t kStage = NMAT * kA + kB;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full_a[kStages], full_b[kStages], empty[kStages], done_bar;
    __shared__ uint32_t tmem_base;
    __shared__ int rows_idx[kTileN];
    // 1024-byte alignment of the swizzled tiles
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    const int tile = blockIdx.x;
    if (tile >= __ldg(g.n_tiles)) return;
    if (*reinterpret_cast<volatile uint32_t*>(g.err)) return;   // an earlier CTA gave up
    const int4 td = __ldg(g.tiles + tile);
    const int row0 = td.x, nrows = td.y, m0 = td.z, slot = td.w;
    const int npad = (nrows + 15) & ~15;
    const int D = g.P.D, F = g.P.F;
    const int K = (MODE == 1) ? D : F;
    const int KT = K / kTileK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_a[s], kDqWarps);
            mbar_init(&full_b[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done_bar, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        const uint32_t ncols = (MODE == 1) ? 512u : 256u;
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    const int tix = (int)threadIdx.x;
    if (tix < kTileN) rows_idx[tix] = tix < nrows ? ((MODE == 1) ? __ldg(g.perm + row0 + tix) : row0 + tix) : -1;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp < kDqWarps) {
        // ---------------- producers of the weight tiles
        const PlanesP<FMT> pl0 = pplanes<FMT>(g.P, slot, MODE == 1 ? 0 : 2);
        const PlanesP<FMT> pl1 = pplanes<FMT>(g.P, slot, 1);
        // 256 threads: MODE 1 -> thread = (matrix, row), 64 weights each per stage;
        //              MODE 2 -> thread = (row, half), 32 weights each per stage.
        const int tid = threadIdx.x;
        for (int j = 0; j < KT; ++j) {
            const int s = j % kStages;
            if (j >= kStages && !mbar_wait(&empty[s], ((j / kStages) - 1) & 1, g.err)) break;
            uint8_t* a_base = smem + (size_t)s * kStage;
            if constexpr (MODE == 1) {
                const int mat = tid >> 7, r = tid & 127;
                const PlanesP<FMT>& pl = mat ? pl1 : pl0;
                uint8_t* at = a_base + mat * kA;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[16];
                    dequant32<FMT>(pl.c, pl.m, pl.d, m0 + r, K, 2 * j + half, pk);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(at + sw128(r, half * 4 + c)) =
                            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
            } else {
                const int r = tid >> 1, half = tid & 1;
                uint32_t pk[16];
                dequant32<FMT>(pl0.c, pl0.m, pl0.d, m0 + r, K, 2 * j + half, pk);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(a_base + sw128(r, half * 4 + c)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            }
            fence_proxy_async();     // make the generic-proxy stores visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_a[s]);
        }
        // ---------------- epilogue: TMEM -> registers -> global
        if (mbar_wait(&done_bar, 0, g.err)) {
            tc_fence_after();
            const int q = warp & 3;                      // TMEM lane quadrant
            const int r = q * 32 + lane;                 // tile row = feature / output index
            const int c_lo = (warp >> 2) * (npad / 2), c_hi = c_lo + npad / 2;
            for (int c = c_lo; c < c_hi; c += 8) {
                const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c;
                float v0[8];
                tmem_ld8(ta, v0);
                if constexpr (MODE == 1) {
                    float v1[8];
                    tmem_ld8(ta + 256, v1);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int n = c + i;
                        if (n < nrows) {
                            const float gte = v0[i], up = v1[i];
                            const float hv = gte / (1.0f + expf(-gte)) * up;
                            g.dst[(size_t)(row0 + n) * F + m0 + r] = f32_to_bf16_rne(hv);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int n = c + i;
                        if (n < nrows) g.dst[(size_t)(row0 + n) * D + m0 + r] = f32_to_bf16_rne(v0[i]);
                    }
                }
            }
        }
    } else if (warp == kGatherWarp) {
        // ---------------- gather of the row operand (K-major, 128B swizzle) with cp.async
        for (int j = 0; j < KT; ++j) {
            const int s = j % kStages;
            if (j >= kStages && !mbar_wait(&empty[s], ((j / kStages) - 1) & 1, g.err)) break;
            const uint32_t b_base = smem_u32(smem + (size_t)s * kStage + NMAT * kA);
            const size_t stride = (size_t)K;
            for (int i = lane; i < npad * 8; i += 32) {
                const int n = i >> 3, c = i & 7;
                const int src_row = rows_idx[n] >= 0 ? rows_idx[n] : rows_idx[0];   // pad rows repeat row 0
                cp_async16(b_base + sw128(n, c), g.src + (size_t)src_row * stride + (size_t)j * kTileK + c * 8);
            }
            cp_async_wait_all();
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_b[s]);
        }
    } else if (warp == kMmaWarp) {
        // ---------------- single-thread MMA issue
        if (lane == 0) {
            const uint32_t idesc = instr_desc(npad);
            bool ok = true;
            for (int j = 0; j < KT && ok; ++j) {
                const int s = j % kStages;
                ok = mbar_wait(&full_a[s], (j / kStages) & 1, g.err) && mbar_wait(&full_b[s], (j / kStages) & 1, g.err);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + (size_t)s * kStage);
                const uint32_t b_addr = a_addr + NMAT * kA;
#pragma unroll
                for (int kk = 0; kk < kTileK / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(b_addr + kk * 32);
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    mma_bf16(tmem, smem_desc_sw128(a_addr + kk * 32), bd, idesc, acc);
                    if constexpr (MODE == 1) mma_bf16(tmem + 256, smem_desc_sw128(a_addr + kA + kk * 32), bd, idesc, acc);
                }
                mma_commit(&empty[s]);     // frees the stage once these MMAs completed
            }
            mma_commit(&done_bar);         // all MMAs of the tile
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        const uint32_t ncols = (MODE == 1) ? 512u : 256u;
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
    }
}

template <int FMT>
moe_status launch_gemms(const PoolView& P, const PrefillWs& w, const uint16_t* x, uint16_t* yrows, int max_t1,
                        int max_t2, cudaStream_t s) {
    const size_t smem1 = (size_t)kStages * (2 * kTileM * kTileK * 2 + kTileN * kTileK * 2) + 1024;
    const size_t smem2 = (size_t)kStages * (kTileM * kTileK * 2 + kTileN * kTileK * 2) + 1024;
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(expert_gemm_kernel<FMT, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
        cudaFuncSetAttribute(expert_gemm_kernel<FMT, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
        attr = true;
    }
    GemmArgs a1;
    a1.P = P; a1.tiles = w.tiles1; a1.n_tiles = w.meta + 1; a1.src = x; a1.perm = w.perm; a1.dst = w.h; a1.err = w.err;
    cudaError_t e = launch_pdl(expert_gemm_kernel<FMT, 1>, dim3(max_t1), dim3(kThreads), smem1, s, a1);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    GemmArgs a2;
    a2.P = P; a2.tiles = w.tiles2; a2.n_tiles = w.meta + 2; a2.src = w.h; a2.perm = nullptr; a2.dst = yrows; a2.err = w.err;
    e = launch_pdl(expert_gemm_kernel<FMT, 2>, dim3(max_t2), dim3(kThreads), smem2, s, a2);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

size_t prefill_workspace_bytes(int T, int D, int F, int E, int k) { return ws_sizes(T, D, F, E, k).total; }

moe_status launch_prefill_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x, int T,
                                  const int32_t* ids, int k, void* expert_out, int32_t* miss_list,
                                  int32_t* miss_count, void* ws, cudaStream_t s) {
    if (P.F % kTileM || P.D % kTileM || E > kMaxE) return MOE_ERR_UNSUPPORTED;
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
    const WsSizes sz = ws_sizes(T, P.D, P.F, E, k);
    const int max_t1 = (int)(sz.t1 / sizeof(int4)), max_t2 = (int)(sz.t2 / sizeof(int4));
    uint16_t* yrows = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(expert_out) + rowmap_bytes(T, k));
    switch (P.fmt) {
        case MOE_Q2_32: return launch_gemms<MOE_Q2_32>(P, w, x, yrows, max_t1, max_t2, s);
        case MOE_Q3_32: return launch_gemms<MOE_Q3_32>(P, w, x, yrows, max_t1, max_t2, s);
        default: return launch_gemms<MOE_Q3_S256>(P, w, x, yrows, max_t1, max_t2, s);
    }
}

}  // namespace moe
