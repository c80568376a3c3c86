// decode.cu — expert pass for 1-8 tokens (one token plus MTP drafts):
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
// Arithmetic: warp-level tensor-core MMAs (mma.sync m16n8k16, fp16 operands,
// fp32 accumulation).  A = 16 weight rows x 16 K, dequantised in registers to
// fp16 (dequant.cuh: each weight the exact weight rounded once to fp16);
// B = 16 K x 8 token columns holding the (up to eight) tokens; columns past T
// are zero.  Every owner is evaluated for all tokens of
// the batch (the tensor cores have the columns to spare) and only the outputs
// of the tokens that selected it are kept, so the cost per weight does not
// depend on how many tokens share an expert.
//
// K order.  Within every 128-K unit U of a row, lane c of a lane quad handles
// the 32-weight block 4U + c; step (i, j) (i = half of the block, j = 0..3)
// gives its A registers the weight pairs (j, j + 8) and (j + 4, j + 12) of
// half i, which one word of codes yields without moving bits (dequant.cuh).
// The MMA's K index 2c + e (e = 0, 1) of step (i, j) is weight
// 128U + 32c + 16i + j + 8e, and 2c + 8 + e is 128U + 32c + 16i + j + 4 + 8e.
// Activations (x, and h for the down projection) are stored in fp16 in that
// order ("fragment order"), so a lane's B registers are one 8-byte load.
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "dequant.cuh"
#include "kernels.cuh"
#include "once.cuh"
#include "route_warp.cuh"
#include "sync.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kTeams = 2;                          // consumer teams, alternating items
constexpr int kTeamWarps = kConsumerWarps / kTeams;
constexpr int kProducerWarp = kConsumerWarps;      // bulk copies into the stage ring
constexpr int kPublisherWarp = kConsumerWarps + 1; // releases finished gate|up items to other CTAs
constexpr int kThreads = kConsumers + 64;
constexpr int kUnitK = 128;
constexpr int kMaxPairs = kDecodeMaxT * kMaxTopK + 1;
constexpr int kMaxStages = 8;
constexpr int kMaxTiles = 2;                       // gate|up 16-row tiles per item (rf <= 16)
// one warp's partial sums of a gate|up item: tiles x (16 rows x NSLOT tokens)
template <int NSLOT>
constexpr int red_floats() { return kMaxTiles * 16 * NSLOT; }
constexpr int kSmemBudget = 220 * 1024;            // dynamic shared memory, at most (see smem_budget)
constexpr int kMaxE = 1024;

// ---------------------------------------------------------------- format geometry
template <int FMT>
struct Geo {
    static constexpr int kBlock = (FMT == MOE_Q3_S256) ? 256 : 32;
    static constexpr int kBlockCode = (FMT == MOE_Q2_32) ? 8 : (FMT == MOE_Q3_32 ? 12 : 96);
    static constexpr int kCb = (FMT == MOE_Q2_32) ? 8 : 12;    // code bytes per 32 weights
    // bytes of one matrix row with K weights, per region
    static constexpr int code_row(int K) { return K / 32 * kCb; }
    static constexpr int meta_row(int K) { return (FMT == MOE_Q3_S256) ? K / 256 * 12 : K / 32 * 4; }
    static constexpr int d_row(int K) { return (FMT == MOE_Q3_S256) ? K / 256 * 2 : 0; }
    static constexpr int row_bytes(int K) { return code_row(K) + meta_row(K) + d_row(K); }
};

// Smallest y >= x with y % m == r.
constexpr uint32_t pad_to(uint32_t x, uint32_t m, uint32_t r) { return x + ((r + m - x % m) % m); }

// A staged region of n matrix rows of K weights: the n code rows, then the n
// meta rows, then (Q3_S256) the n d rows, each plane at its own smem row
// stride.  Code and Q2/Q3_32 scale rows are copied one row at a time into
// padded rows, so that the eight rows read by one load instruction (lanes g =
// 0..7, four lanes a row) fall on distinct banks:
//   Q2 codes      8-byte loads, 32 bytes a row:  stride = 32 (mod 64)
//   Q3 codes      three 4-byte loads, 12 bytes a lane: stride = 16 (mod 32)
//   (s, m) words  4-byte loads, 16 bytes a row:  stride = 16 (mod 32)
// (rows r * stride then start at distinct 32-byte (resp. 16-byte) slots of the
// 128-byte bank window, since stride / 16 is odd).  The Q3_S256 sub-scale and
// d rows are read with broadcasts (one super-block a row) and copied unpadded
// in one piece.
template <int FMT>
struct Rows {
    uint32_t c, m, d;     // smem row strides of the planes
    uint32_t cr, mr, dr;  // bytes of one row in the pool (padding: zeros past cr, mr)
    static constexpr Rows of(int K) {
        Rows R{};
        R.cr = Geo<FMT>::code_row(K);
        R.mr = Geo<FMT>::meta_row(K);
        R.dr = Geo<FMT>::d_row(K);
        R.c = FMT == MOE_Q2_32 ? pad_to(R.cr, 64, 32) : pad_to(R.cr, 32, 16);
        R.m = FMT == MOE_Q3_S256 ? R.mr : pad_to(R.mr, 32, 16);
        R.d = R.dr;
        return R;
    }
    constexpr uint32_t bytes(int n) const { return (uint32_t)n * (c + m + d); }      // staged (and copied)
    constexpr uint32_t region(int n) const { return (bytes(n) + 127u) & ~127u; }     // 128-byte aligned slot
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

// One stage of the ring: a gate|up item (gate rows, then up rows, each in a
// 128-byte aligned region) or a down item (rows, then the owner's h), 128-byte
// aligned (tensor copies land on 128-byte boundaries).
template <int FMT, int NSLOT>
constexpr uint32_t stage_size(int D, int F, int rf, int rd) {
    const uint32_t a = 2u * Rows<FMT>::of(D).region(rf);
    const uint32_t b = Rows<FMT>::of(F).bytes(rd) + (uint32_t)F * NSLOT * 2;
    return ((a > b ? a : b) + 127u) & ~127u;
}

// ---------------------------------------------------------------- work resolution
struct Owner {
    int slot;
    uint32_t rmask[kDecodeMaxT];   // ranks of token t served by this expert (0: token not served)
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
    int t0;                // the batch's first token in the caller's batch (rowmap, yrows: already offset)
    int miss_append;       // 1: misses follow those already counted in miss_count (a batch's second launch)
    uint16_t* hfrag;       // [kMaxPairs][F * NSLOT] fp16, fragment order
    uint32_t* err;
    uint32_t* done;        // [kMaxPairs + 2]: per-owner gate|up completion counters, CTA ticket, work queue
    int rf;                // gate|up: features per item (8 or 16)
    int rd;                // down: rows per item (multiple of 16)
    int ns;                // pipeline stages
    // padded-row boxes (Rows<FMT>): gate|up matrices as one tensor of 2F rows
    // of D weights, down as D rows of F weights; codes and (s, m) planes
    // (Q3_S256: the code maps only)
    CUtensorMap tm_gu_c, tm_gu_m, tm_dn_c, tm_dn_m;
    // the one-call layer (moe_layer_forward): routing in the kernel, combine
    // at the end (unused otherwise)
    const uint16_t* Wr;    // [E][D] bf16
    const float* bias;     // [E] or null
    int route_j;           // experts whose logits each CTA computes (CTA b: route_j * b + j)
    int route_wr_smem;     // 1: those Wr rows are copied into the stage ring (after x), else read from L2
    float* logits;         // [T][E] fp32 scratch
    int32_t* ids_out;      // [T][k]
    float* gates_out;      // [T][k]
    const uint16_t* residual;   // [T][D] bf16 or null
    uint16_t* out;         // [T][D] bf16
};

constexpr int kRedBufs = 3;                        // partial-sum buffers per team (items in flight)
constexpr int kPubRing = 64;                       // finished gate|up items awaiting release
constexpr uint32_t kPubEnd = 0xffffffffu;          // ring entry: no more items (others: owner + 1)

struct Shared {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    int stage_item[kMaxStages];    // the work item in each stage (-1: no more work)
    Owner owners[kMaxPairs];
    int table[kMaxE];              // the slot table, staged before the dependency wait
    int oidx[kMaxPairs];           // per owning pair: its owner index
    int n_owners;
    int abort;                     // set by any warp that stopped on an error
    uint32_t red_cnt[kTeams][kRedBufs];   // warps that wrote their partials into a buffer
    uint32_t red_gen[kTeams][kRedBufs];   // reductions completed on a buffer
    uint32_t pub_head;             // finished gate|up items queued for the publisher
    int pubq[kPubRing];            // their owners + 1 (0: free; kPubEnd: no more items)
    uint32_t finished;             // warps (consumers, producer) that are done
    int32_t sids[kDecodeMaxT * kMaxTopK];   // one-call layer: the selected ids and gates
    float sgates[kDecodeMaxT * kMaxTopK];
    float sbias[kConsumerWarps];    // the router bias of this CTA's logit experts
};

// The slot table is an input of the layer, not produced by the router: stage it
// while the router may still run.
// `first` (E ints, scratch for resolve_owners) starts at kMaxPairs.
__device__ void stage_table(const DecodeParams& prm, Shared& sh, int* first) {
    for (int e = threadIdx.x; e < prm.E; e += blockDim.x) {
        const int s = __ldg(prm.slot_table + e);
        sh.table[e] = (s < 0 || s >= prm.P.n_slots) ? -1 : s;
        first[e] = kMaxPairs;
    }
}

// Work items: owner u's gate|up items are nfb = F / rf blocks of rf features,
// its down items nrb = D / rd blocks of rd output rows; item i of a phase
// belongs to owner i / per_owner.
struct ItemPos { int u, row0; };
MOE_DEVINL ItemPos item_pos(int i, int per_owner, int rows) {
    ItemPos p;
    p.u = i / per_owner;
    p.row0 = (i - p.u * per_owner) * rows;
    return p;
}

MOE_DEVINL int lookup_slot(const DecodeParams& prm, const Shared& sh, int e) {
    return (e >= 0 && e < prm.E) ? sh.table[e] : -1;
}

// One warp: resolve every pair's slot and the owners — owner 0 is the shared
// expert, then the first pair of each distinct resident expert in pair order —
// and, with `book`, the row map, miss list and miss count.  The ids come
// from global memory (prm.ids) or, in the one-call layer, from shared memory
// (ids_smem).  Lane L handles
// pairs L + 32h (h = 0..3; T * k <= 128).  Pairs of one expert find their
// owner through a shared-memory minimum per expert id (`first`: E ints, all
// kMaxPairs on entry); each pair then sets its rank bit in its owner's token
// mask.  (Two expert ids on one slot would get
// two owners over the same weights: the same outputs, computed twice.)
__device__ void resolve_owners(const DecodeParams& prm, Shared& sh, int* first, bool book,
                               const int32_t* ids_smem) {
    constexpr int H = (kMaxPairs - 1 + 31) / 32;
    const int lane = threadIdx.x & 31;
    const int T = prm.T, k = prm.k, n = T * k;   // n <= 128
    const int hn = (n + 31) >> 5;                // pair groups in use (warp-uniform)
    const uint32_t below = (1u << lane) - 1u;
    int e[H], s[H], tt[H], rr[H];
    uint32_t missb[H];
#pragma unroll
    for (int h = 0; h < H; ++h) {
        const int p = lane + 32 * h;
        e[h] = h < hn && p < n ? (ids_smem ? ids_smem[p] : __ldg(prm.ids + p)) : -1;
        tt[h] = p / k;
        rr[h] = p - tt[h] * k;
    }
#pragma unroll
    for (int h = 0; h < H; ++h) {
        if (h >= hn) break;
        const int p = lane + 32 * h;
        s[h] = p < n ? lookup_slot(prm, sh, e[h]) : -1;
        if (s[h] >= 0) atomicMin(first + e[h], p);
        missb[h] = __ballot_sync(0xffffffffu, p < n && s[h] < 0);
    }
    if (book) {
        // row-map values and miss tokens are the caller's batch indices (t0 + t); a
        // batch's second launch appends its misses after the first launch's
        const int t0 = prm.t0;
        int base = prm.miss_append ? *reinterpret_cast<volatile const int32_t*>(prm.miss_count) : 0;
#pragma unroll
        for (int h = 0; h < H; ++h) {
            if (h >= hn) break;
            const int p = lane + 32 * h;
            if (p < n) {
                const int t = tt[h], r = rr[h];
                prm.rowmap[t * (k + 1) + r] = s[h] >= 0 ? (t0 + t) * (k + 1) + r : -1;
                if (s[h] < 0) {
                    const int pos = base + __popc(missb[h] & below);
                    prm.miss_list[3 * pos + 0] = t0 + t; prm.miss_list[3 * pos + 1] = r; prm.miss_list[3 * pos + 2] = e[h];
                }
            }
            base += __popc(missb[h]);
        }
        if (lane < T) prm.rowmap[lane * (k + 1) + k] = (t0 + lane) * (k + 1) + k;
        __syncwarp();                                 // every lane has read the count before lane 0 rewrites it
        if (lane == 0) prm.miss_count[0] = base;
    }
    __syncwarp();
    int base = 1;
#pragma unroll
    for (int h = 0; h < H; ++h) {
        if (h >= hn) break;
        const int p = lane + 32 * h;
        const bool own = s[h] >= 0 && first[e[h]] == p;
        const uint32_t ownb = __ballot_sync(0xffffffffu, own);
        if (own) {
            const int o = base + __popc(ownb & below);
            sh.oidx[p] = o;
            sh.owners[o].slot = s[h];
#pragma unroll
            for (int t = 0; t < kDecodeMaxT; ++t) sh.owners[o].rmask[t] = 0u;
        }
        base += __popc(ownb);
    }
    if (lane < kDecodeMaxT) sh.owners[0].rmask[lane] = lane < T ? 1u << k : 0u;
    if (lane == 0) {
        sh.owners[0].slot = prm.P.shared_slot;
        sh.n_owners = base;
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < H; ++h) {
        if (h >= hn) break;
        if (s[h] >= 0) atomicOr(&sh.owners[sh.oidx[first[e[h]]]].rmask[tt[h]], 1u << rr[h]);
    }
    __syncwarp();
}

// ---------------------------------------------------------------- activations in fragment order
// Byte offset of the 8-byte B-register pair of step s = (U * 2 + i) * 4 + j,
// token column n, lane-in-quad c.
template <int NSLOT>
MOE_DEVINL uint32_t frag_off(int step, int n, int c) { return (uint32_t)(((step * NSLOT + n) * 4 + c) * 8); }

// 16 consecutive bf16 values of one token (a half block) as fp16 in fragment
// order: four 8-byte words (j = 0..3), each (v[j], v[j + 8]) in the low word
// and (v[j + 4], v[j + 12]) in the high word.  Returns false if a value is
// outside the fp16 range.
MOE_DEVINL bool half_block_frag(const uint4 a, const uint4 b, uint2 (&out)[4]) {
    float v[16];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) { v[2 * q] = bf16lo(w[q]); v[2 * q + 1] = bf16hi(w[q]); }
    bool ok = true;
#pragma unroll
    for (int q = 0; q < 16; ++q) ok &= fabsf(v[q]) < 65520.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) out[j] = make_uint2(pack_f16x2(v[j], v[j + 8]), pack_f16x2(v[j + 4], v[j + 12]));
    return ok;
}

// x [T][K] (bf16, global) -> xs (fp16 fragment order, NSLOT token columns;
// columns >= T zero).  Run by `nthreads` threads starting at thread `first`.
template <int NSLOT>
__device__ void stage_x_frag(const uint16_t* __restrict__ x, int T, int K, uint8_t* xs, uint32_t* err, int first,
                             int nthreads, uint16_t* xcopy = nullptr) {
    const int nhb = K / 16, total = NSLOT * nhb;
    bool ok = true;
    // two half blocks per thread and round, both loads in flight before the stores
    for (int idx0 = (int)threadIdx.x - first; idx0 < total; idx0 += 2 * nthreads) {
        uint4 a[2], b[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int idx = idx0 + q * nthreads, n = idx / nhb, hb = idx - n * nhb;
            a[q] = b[q] = make_uint4(0, 0, 0, 0);
            if (idx < total && n < T) {
                const uint4* p = reinterpret_cast<const uint4*>(x + (size_t)n * K + 16 * hb);
                a[q] = __ldg(p);
                b[q] = __ldg(p + 1);
            }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int idx = idx0 + q * nthreads, n = idx / nhb, hb = idx - n * nhb;
            if (idx >= total) continue;
            uint2 o[4] = {make_uint2(0, 0), make_uint2(0, 0), make_uint2(0, 0), make_uint2(0, 0)};
            if (n < T) {
                ok &= half_block_frag(a[q], b[q], o);
                if (xcopy) {             // and the rows as they are (bf16 [T][K])
                    uint4* c = reinterpret_cast<uint4*>(xcopy + (size_t)n * K + 16 * hb);
                    c[0] = a[q];
                    c[1] = b[q];
                }
            }
            // hb = U * 8 + c * 2 + i
            const int U = hb >> 3, c = (hb >> 1) & 3, i = hb & 1;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint2*>(xs + frag_off<NSLOT>((U * 2 + i) * 4 + j, n, c)) = o[j];
        }
    }
    if (!ok) atomicOr(err, kErrRange);
}

// Halfword index of element (kk, token n) in a fragment-order buffer.
template <int NSLOT>
MOE_DEVINL uint32_t frag_half_index(int kk, int n) {
    const int U = kk >> 7, c = (kk >> 5) & 3, i = (kk >> 4) & 1, o = kk & 15;
    const int j = o & 3, breg = (o >> 2) & 1, e = o >> 3;
    return (uint32_t)((((U * 2 + i) * 4 + j) * NSLOT + n) * 4 + c) * 4 + (uint32_t)(breg * 2 + e);
}

// ---------------------------------------------------------------- MMA
MOE_DEVINL void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One row's data for the 32-weight block of a lane in one 128-K unit: the
// code words and the block scales.
template <int FMT>
struct RowBlock {
    uint32_t w[3];           // code words (Q2: w[0], w[1] = halves 0, 1)
    uint32_t sa, sb;         // Q2/Q3_32: s and m broadcast to f16x2; Q3_S256: sc - 32 of halves 0 and 1
    uint32_t d2;             // Q3_S256: d broadcast to f16x2
};

// Load block (4U + c) of local row r of a staged region (planes at cbase,
// mbase, dbase; row strides R).
template <int FMT>
MOE_DEVINL void load_row_block(const uint8_t* cbase, const uint8_t* mbase, const uint8_t* dbase, int r,
                               const Rows<FMT>& R, int U, int c, RowBlock<FMT>& rb) {
    const int blk = 4 * U + c;
    if constexpr (FMT == MOE_Q2_32) {
        const uint2 v = *reinterpret_cast<const uint2*>(cbase + (size_t)r * R.c + blk * 8);
        rb.w[0] = v.x; rb.w[1] = v.y; rb.w[2] = 0;
    } else {
        const uint32_t* p = reinterpret_cast<const uint32_t*>(cbase + (size_t)r * R.c + blk * 12);
        rb.w[0] = p[0]; rb.w[1] = p[1]; rb.w[2] = p[2];
    }
    if constexpr (FMT != MOE_Q3_S256) {
        const uint32_t sm = *reinterpret_cast<const uint32_t*>(mbase + (size_t)r * R.m + blk * 4);
        rb.sa = bcast_lo(sm);
        rb.sb = bcast_hi(sm);
        rb.d2 = 0;
    } else {
        // super-block U / 2; the block's two sub-blocks: 12 bits at bit 12 * (4 (U & 1) + c)
        const uint32_t* scp = reinterpret_cast<const uint32_t*>(mbase + (size_t)r * R.m + (U >> 1) * 12);
        const int cc = 4 * (U & 1) + c, bit = 12 * cc, wi = bit >> 5, sh = bit & 31;
        const uint32_t lo = scp[wi];
        const uint32_t hi = wi < 2 ? scp[wi + 1] : 0u;
        const uint32_t bits = __funnelshift_r(lo, hi, sh);
        const uint32_t db = *reinterpret_cast<const uint16_t*>(dbase + (size_t)r * R.d + (U >> 1) * 2);
        rb.d2 = db | (db << 16);
        rb.sa = s256_sub(bits & 63u);
        rb.sb = s256_sub((bits >> 6) & 63u);
    }
}

// Weight pairs (j, j + 8) and (j + 4, j + 12) of half I, the A registers of
// step (I, J) for one row.
template <int FMT, int I, int J>
MOE_DEVINL void step_pairs(const RowBlock<FMT>& rb, const Magic& M, uint32_t& lo, uint32_t& hi) {
    if constexpr (FMT == MOE_Q2_32) {
        const uint32_t w = rb.w[I], w10 = w >> 10;
        lo = w_sm(q2_codes<J>(w, w10, M), rb.sa, rb.sb);
        hi = w_sm(q2_codes<J + 4>(w, w10, M), rb.sa, rb.sb);
    } else {
        uint32_t P, P2;
        q3_group_words(rb.w[0], rb.w[1], rb.w[2], I, P, P2);
        const uint32_t P9 = P >> 9, P10 = P2 >> 10;
        if constexpr (FMT == MOE_Q3_32) {
            lo = w_sm(q3_codes<J, false>(P, P9, P2, P10, M), rb.sa, rb.sb);
            hi = w_sm(q3_codes<J + 4, false>(P, P9, P2, P10, M), rb.sa, rb.sb);
        } else {
            const uint32_t sc2 = I == 0 ? rb.sa : rb.sb;
            lo = w_s256(q3_codes<J, true>(P, P9, P2, P10, M), sc2, rb.d2);
            hi = w_s256(q3_codes<J + 4, true>(P, P9, P2, P10, M), sc2, rb.d2);
        }
    }
}

// Compile-time loop: f(std::integral_constant<int, I>) for I in [B, E).
template <int B, int E, typename Fn>
MOE_DEVINL void static_for(Fn&& fn) {
    if constexpr (B < E) {
        fn(std::integral_constant<int, B>{});
        static_for<B + 1, E>(fn);
    }
}

// One 128-K unit U for NT tiles: tile t's A rows g and g + 8 are local rows
// rt[t] of region (ca, ma, da) and rbm[t] of region (cb, mb, db); B from the
// fragment-order buffer bs.  Accumulates into acc[t].
template <int FMT, int NT, int NSLOT>
MOE_DEVINL void unit_mma(const uint8_t* ca, const uint8_t* ma, const uint8_t* da, const uint8_t* cb,
                         const uint8_t* mb, const uint8_t* db, const int (&rt)[NT], const int (&rbm)[NT],
                         const Rows<FMT>& R, int U, const uint8_t* bs, const Magic& M, float (&acc)[NT][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    RowBlock<FMT> top[NT], bot[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        load_row_block<FMT>(ca, ma, da, rt[t], R, U, c, top[t]);
        load_row_block<FMT>(cb, mb, db, rbm[t], R, U, c, bot[t]);
    }
    static_for<0, 8>([&](auto S) {
        constexpr int s = decltype(S)::value, I = s >> 2, J = s & 3;
        uint32_t b0 = 0, b1 = 0;
        if (g < NSLOT) {
            const uint2 bv = *reinterpret_cast<const uint2*>(bs + frag_off<NSLOT>(U * 8 + s, g, c));
            b0 = bv.x;
            b1 = bv.y;
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            uint32_t a[4];
            step_pairs<FMT, I, J>(top[t], M, a[0], a[2]);
            step_pairs<FMT, I, J>(bot[t], M, a[1], a[3]);
            mma16816(acc[t], a, b0, b1);
        }
    });
}

MOE_DEVINL float silu_f(float g) { return g / (1.0f + expf(-g)); }

// The copies of `nrows` rows starting at row y of a matrix set (tensor maps
// mc, mm over the slot's rows; pl: the slot's planes of the matrix, rows from
// row0) into the region at dst (layout Rows<FMT>), completing on bar: one
// padded-row box per code and (s, m) plane; the Q3_S256 sub-scale and d planes
// in one bulk copy each.  Every copied byte, padding included, counts toward
// the barrier's transaction bytes: Rows<FMT>::bytes(nrows).
template <int FMT>
MOE_DEVINL void issue_rows(const CUtensorMap* mc, const CUtensorMap* mm, const Planes& pl, int y, int row0,
                           int slot, int nrows, const Rows<FMT>& R, uint8_t* dst, uint64_t* bar) {
    tma_box_3d(dst, mc, 0, y, slot, bar);
    uint8_t* dm = dst + (size_t)nrows * R.c;
    if constexpr (FMT != MOE_Q3_S256) {
        (void)pl; (void)row0;
        tma_box_3d(dm, mm, 0, y, slot, bar);
    } else {
        (void)mm;
        bulk_g2s(dm, pl.m + (size_t)row0 * R.mr, R.mr * nrows, bar);
        bulk_g2s(dm + (size_t)nrows * R.m, pl.d + (size_t)row0 * R.dr, R.dr * nrows, bar);
    }
}

// ---------------------------------------------------------------- gate | up
// Item = (owner u, features [f0, f0 + rf)), staged as gate rows then up rows.
// 16-row MMA tile t: rows g = gate feature 8t + g, rows g + 8 = up feature
// 8t + g, so the lane holding the gate value of (feature, token) also holds
// the up value.  The eight warps of the team split K by 128-K units; their
// partial sums meet in `red_w` (this warp's slot), and the team's warp 0 forms h.
template <int FMT, int NT, int NSLOT>
__device__ void gateup_partial(const DecodeParams& prm, int rf, const uint8_t* stage, const uint8_t* xs, int wt,
                               float* red_w) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int D = prm.P.D;
    const Rows<FMT> R = Rows<FMT>::of(D);
    const uint8_t* gc = stage;                     // gate rows, then up rows
    const uint8_t* gm = gc + R.c * rf;
    const uint8_t* gd = gm + R.m * rf;
    const uint8_t* uc = stage + R.region(rf);
    const uint8_t* um = uc + R.c * rf;
    const uint8_t* ud = um + R.m * rf;
    const Magic M = make_magic();
    float acc[NT][4];
    int rt[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        rt[t] = 8 * t + g;
        acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    }
    for (int U = wt; U < D / kUnitK; U += kTeamWarps)
        unit_mma<FMT, NT, NSLOT>(gc, gm, gd, uc, um, ud, rt, rt, R, U, xs, M, acc);
    // lanes with c < NSLOT / 2 hold token columns 2c, 2c + 1 (the columns in use)
    if (c < NSLOT / 2) {
#pragma unroll
        for (int t = 0; t < NT; ++t)
            *reinterpret_cast<float4*>(red_w + (t * 8 * (NSLOT / 2) + g * (NSLOT / 2) + c) * 4) =
                make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
    }
}

// The team's warp 0: sum the eight partials of every (feature, token) in warp
// order, h = bf16(silu(gate) * up), stored as fp16 in the owner's
// fragment-order h buffer.  Entry q = (tile, g, c) of the partials holds
// gate and up of feature 8 tile + g for tokens 2c and 2c + 1.
template <int NSLOT>
__device__ void gateup_reduce(const DecodeParams& prm, int u, int f0, int rf, const float* red) {
    const int lane = threadIdx.x & 31;
    constexpr int kC = NSLOT / 2;                 // lanes in use per row group
    const int nq = (rf / 8) * 8 * kC;             // entries
    const int F = prm.P.F;
    uint16_t* hf = prm.hfrag + (size_t)u * F * NSLOT;
    bool ok = true;
    for (int q = lane; q < nq; q += 32) {
        const int t = q / (8 * kC), g = (q / kC) & 7, c = q % kC;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kTeamWarps; ++w) {
            const float4 v = *reinterpret_cast<const float4*>(red + w * red_floats<NSLOT>() + q * 4);
            s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
        }
        const int f = f0 + 8 * t + g;
        const float hv0 = bf16_bits_to_f32(f32_to_bf16_rne(silu_f(s.x) * s.z));   // token 2c
        const float hv1 = bf16_bits_to_f32(f32_to_bf16_rne(silu_f(s.y) * s.w));   // token 2c + 1
        ok &= fabsf(hv0) < 65520.f && fabsf(hv1) < 65520.f;
        hf[frag_half_index<NSLOT>(f, 2 * c)] = __half_as_ushort(__float2half_rn(hv0));
        hf[frag_half_index<NSLOT>(f, 2 * c + 1)] = __half_as_ushort(__float2half_rn(hv1));
    }
    if (!ok) atomicOr(prm.err, kErrRange);
}

// ---------------------------------------------------------------- down
// Item = (owner u, rows [d0, d0 + rd)) of Wd; warp wt takes the 16-row tile wt
// over the whole K = F.
template <int FMT, int NSLOT>
__device__ void down_item(const DecodeParams& prm, const Owner& o, int d0, int rd, const uint8_t* stage,
                          const uint8_t* hs, int wt) {
    if (16 * wt >= rd) return;
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int D = prm.P.D, F = prm.P.F, k = prm.k;
    const Rows<FMT> R = Rows<FMT>::of(F);
    const uint8_t* dc = stage;
    const uint8_t* dm = dc + R.c * rd;
    const uint8_t* dd = dm + R.m * rd;
    const Magic M = make_magic();
    float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
    const int rt[1] = {16 * wt + g}, rbm[1] = {16 * wt + g + 8};
    for (int U = 0; U < F / kUnitK; ++U) unit_mma<FMT, 1, NSLOT>(dc, dm, dd, dc, dm, dd, rt, rbm, R, U, hs, M, acc);
    if (c < NSLOT / 2) {
        const int row = d0 + 16 * wt + g;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t m = o.rmask[2 * c + h];
            while (m) {
                const int r = __ffs(m) - 1;
                m &= m - 1;
                float* dst = prm.yrows + ((size_t)(2 * c + h) * (k + 1) + r) * D + row;
                dst[0] = acc[0][h];
                dst[8] = acc[0][2 + h];
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
MOE_DEVINL uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ---------------------------------------------------------------- the fused kernel
// One persistent CTA per SM.  Work items come from one queue shared by all
// CTAs (an atomic counter): first the gate|up items of every owner (owner by
// owner), then the down items (owner by owner).  A CTA's producer warp takes
// the next item whenever a stage is free, so the CTAs finish within about one
// item of each other, and by the time a down item of owner u is taken, the
// gate|up items of u were taken long before.  A down item needs the owner's h:
// the producer waits for the owner's gate|up count (a per-owner counter in ws,
// advanced at gpu scope by the publisher warp of whichever CTA finished the
// item) and copies h into the stage after the weights.  Consumer warps never
// wait on each other: each warp of a gate|up item adds its partial sums to the
// team's buffer, and the last one to do so reduces them and queues the item for
// the publisher.  The last CTA to finish resets the counters, so every
// completed call leaves them zero.
// ---------------------------------------------------------------- one-call layer
// The 512 consumer threads meet at named barrier 5.
MOE_DEVINL void consumers_sync() { asm volatile("bar.sync 5, %0;" ::"n"(kConsumers) : "memory"); }

// Queue one entry for the publisher warp (one lane): waits (bounded) for the
// ring slot to be free, then releases the entry (with the caller's prior
// writes, ordered before it by the caller's __syncwarp).
MOE_DEVINL void pub_push(Shared& sh, uint32_t v) {
    const uint32_t pos = atomicAdd(&sh.pub_head, 1u);
    uint32_t* slot = reinterpret_cast<uint32_t*>(&sh.pubq[pos % kPubRing]);
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_cta(slot) != 0u && globaltimer_ns() - t0 < kWaitLimitNs) {}
    st_release_cta(slot, v);
}

// Byte offset of the routing Wr rows in the stage ring (after x, bf16 [T][D]).
__host__ __device__ constexpr size_t wr_ring_offset(int T, int D) { return ((size_t)T * D * 2 + 127) & ~(size_t)127; }

// Grid-wide barrier over one counter (thread 0 of each CTA; every CTA of the
// grid is resident: one CTA per SM).  False, with the timeout bit set, if the
// other CTAs did not all arrive within the wait limit.
MOE_DEVINL bool grid_arrive_wait(uint32_t* count, uint32_t* err) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(count) : "memory");
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(count) < gridDim.x) {
        if (timed_out(err) || globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
    return true;
}

// Routing inside the expert-pass kernel, by the consumer warps of every CTA:
// x staged in fp16 fragment order for the expert pass and, as it is (bf16), in
// the stage ring for the logits; the logits of this CTA's experts route_j * b + j (warp j, the
// router's canonical order and bias; their Wr rows copied into the ring after
// x before the dependency wait, completing on wbar, or read from L2 when they
// do not fit); a grid-wide barrier; then every CTA selects every token's top-k
// itself (the router's selection) into shared memory, and CTA 0 writes the
// ids and gates.  Returns false (on every consumer thread) when a wait gave
// up: the CTA then does no expert work, and CTA 0 writes ids -1 and gates 0.
template <int NSLOT>
__device__ bool route_phase(const DecodeParams& prm, Shared& sh, uint8_t* xs, uint8_t* ring, uint64_t* wbar,
                            bool rows_issued, uint32_t* grid_count) {
    const int warp = threadIdx.x >> 5;
    const int T = prm.T, D = prm.P.D, E = prm.E, k = prm.k, J = prm.route_j;
    uint16_t* xb = reinterpret_cast<uint16_t*>(ring);
    const uint16_t* wsm = reinterpret_cast<const uint16_t*>(ring + wr_ring_offset(T, D));
    stage_x_frag<NSLOT>(prm.x, T, D, xs, prm.err, 0, kConsumers, xb);
    __shared__ int x_ok;
    if (threadIdx.x == 0) {
        bool ok = true;
        if (rows_issued) {
            ok = mbar_wait(wbar, 0, prm.err);
            if (!ok) mbar_drain(wbar, 0);        // the copy lands before the ring is reused
        }
        x_ok = ok;
    }
    consumers_sync();
    // one (expert, token) logit per warp at a time: the per-token sums are
    // independent, so spreading them over the warps keeps the canonical order
    for (int q = warp; x_ok && q < J * T; q += kConsumerWarps) {
        const int j = q % J, t = q / J, e = J * (int)blockIdx.x + j;
        if (e >= E) continue;
        if (prm.route_wr_smem)
            canon_logits_warp_xbf16<1, true>(xb + (size_t)t * D, 1, D, wsm + (size_t)j * D, prm.bias != nullptr,
                                             sh.sbias[j], E, e, prm.logits + (size_t)t * E);
        else
            canon_logits_warp_xbf16<1, false>(xb + (size_t)t * D, 1, D, prm.Wr + (size_t)e * D, prm.bias != nullptr,
                                              sh.sbias[j], E, e, prm.logits + (size_t)t * E);
    }
    // generic reads of the ring precede the bulk copies that land there later
    fence_proxy_async();
    consumers_sync();
    __shared__ int routed;           // one decision for the whole CTA
    if (threadIdx.x == 0) routed = grid_arrive_wait(grid_count, prm.err) && !timed_out(prm.err) ? 1 : 0;
    consumers_sync();
    if (!routed) {
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i < T * k; i += kConsumers) { prm.ids_out[i] = -1; prm.gates_out[i] = 0.f; }
        return false;
    }
    if (warp < T) topk_warp(prm.logits + (size_t)warp * E, E, k, sh.sids + warp * k, sh.sgates + warp * k);
    consumers_sync();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < T * k; i += kConsumers) { prm.ids_out[i] = sh.sids[i]; prm.gates_out[i] = sh.sgates[i]; }
    return true;
}

// The gate-weighted combine of this CTA's slice of the outputs, after every
// expert row is written: task i = (t, feature pair 2q) of the T * D / 2 tasks,
// CTA b taking a contiguous range; each sums its two features in
// moe_combine's order (hit ranks ascending with fmaf, then the shared expert,
// then the residual), rounds to bf16 and writes out.  Every row of a task is
// loaded before the sums (one round trip); rows written by other CTAs are read
// from L2.
__device__ void combine_slice(const DecodeParams& prm, const Shared& sh) {
    const int T = prm.T, D = prm.P.D, k = prm.k, half = D / 2;
    const int total = T * half, per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int end = min(total, ((int)blockIdx.x + 1) * per);
    const float* rows = prm.yrows;
    for (int task = (int)blockIdx.x * per + (int)threadIdx.x; task < end; task += (int)blockDim.x) {
        const int t = task / half, d = 2 * (task - t * half);
        float2 y[kMaxTopK];
        bool hit[kMaxTopK];
#pragma unroll
        for (int r = 0; r < kMaxTopK; ++r) {
            hit[r] = r < k && lookup_slot(prm, sh, sh.sids[t * k + r]) >= 0;
            y[r] = hit[r] ? __ldcg(reinterpret_cast<const float2*>(rows + (size_t)(t * (k + 1) + r) * D + d))
                          : make_float2(0.f, 0.f);
        }
        const float2 ys = __ldcg(reinterpret_cast<const float2*>(rows + (size_t)(t * (k + 1) + k) * D + d));
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxTopK; ++r) {
            if (hit[r]) {
                const float g = sh.sgates[t * k + r];
                a0 = __fmaf_rn(g, y[r].x, a0);
                a1 = __fmaf_rn(g, y[r].y, a1);
            }
        }
        a0 += ys.x; a1 += ys.y;
        if (prm.residual) {
            const uint32_t rv = *reinterpret_cast<const uint32_t*>(prm.residual + (size_t)t * D + d);
            a0 += bf16lo(rv); a1 += bf16hi(rv);
        }
        *reinterpret_cast<uint32_t*>(prm.out + (size_t)t * D + d) =
            (uint32_t)f32_to_bf16_rne(a0) | ((uint32_t)f32_to_bf16_rne(a1) << 16);
    }
}

template <int FMT, int NSLOT, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1) decode_ffn_kernel(const __grid_constant__ DecodeParams prm) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ Shared sh;
    // tensor copies land on 128-byte boundaries (the launch adds 128 bytes)
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = prm.P.D, F = prm.P.F, rf = prm.rf, rd = prm.rd, NS = prm.ns;
    const size_t xs_bytes = (size_t)D * NSLOT * 2;
    const uint32_t hbytes = (uint32_t)F * NSLOT * 2;                           // one owner's h
    const size_t red_team = (size_t)kRedBufs * kTeamWarps * red_floats<NSLOT>();
    uint8_t* xs = smem;
    float* red = reinterpret_cast<float*>(smem + xs_bytes);
    uint8_t* stages = smem + xs_bytes + kTeams * red_team * 4;
    const Rows<FMT> RD = Rows<FMT>::of(D), RF = Rows<FMT>::of(F);
    const uint32_t dn_bytes = RF.bytes(rd);                                    // down rows, then h
    const uint32_t stage_bytes = stage_size<FMT, NSLOT>(D, F, rf, rd);         // gate rows | up rows
    const int nfb = F / rf, nrb = D / rd;
    uint32_t* done = prm.done;
    uint32_t* queue = done + kMaxPairs + 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], kTeamWarps); }
        fence_mbar_init();
        sh.abort = 0;
        sh.pub_head = 0;
        sh.finished = 0;
        for (int tm = 0; tm < kTeams; ++tm)
            for (int b = 0; b < kRedBufs; ++b) { sh.red_cnt[tm][b] = 0; sh.red_gen[tm][b] = 0; }
    }
    for (int i = threadIdx.x; i < kPubRing; i += blockDim.x) sh.pubq[i] = 0;
    // a call on a workspace whose timeout bit is set does no work (every CTA
    // still takes its ticket below, so the counters are left zero); one read,
    // shared by the whole CTA, so that every warp takes the same branch.  The
    // word is read before the dependency wait: only this kernel writes it, and
    // its previous launch on the stream completed before the router that
    // precedes this launch passed its own wait.
    // (one-call layer: the word is read after the dependency wait, since the
    // previous launch on the workspace may still run until then)
    __shared__ int dead;
    if (!FUSED && threadIdx.x == 0) dead = timed_out(prm.err) ? 1 : 0;
    // the partial-sum buffers are free until the first item: owner resolution
    // keeps its per-expert scratch there
    int* first = reinterpret_cast<int*>(red);
    stage_table(prm, sh, first);
    // one-call layer: this CTA's Wr rows (weights, not produced by the
    // preceding kernel) are prefetched into L2 before the wait, and the bias of
    // each logit warp's expert is loaded
    __shared__ uint64_t wbar;
    const int e0 = prm.route_j * (int)blockIdx.x;
    const bool rows_issued = FUSED && prm.route_wr_smem && min(prm.route_j, prm.E - e0) > 0;
    if constexpr (FUSED) {
        const int nrows = min(prm.route_j, prm.E - e0);
        if (threadIdx.x == 0) {
            mbar_init(&wbar, 1);
            fence_mbar_init();
            if (rows_issued) {
                mbar_arrive_expect_tx(&wbar, (uint32_t)nrows * D * 2u);
                bulk_g2s(stages + wr_ring_offset(prm.T, D), prm.Wr + (size_t)e0 * D, (uint32_t)nrows * D * 2u, &wbar);
            } else if (nrows > 0) {
                prefetch_l2(prm.Wr + (size_t)e0 * D, (uint32_t)nrows * D * 2u);
            }
        }
        if (threadIdx.x < prm.route_j)
            sh.sbias[threadIdx.x] = e0 + (int)threadIdx.x < prm.E && prm.bias ? __ldg(prm.bias + e0 + threadIdx.x) : 0.f;
    }
    __syncthreads();
    pdl_wait();                      // ids come from the router (x: from the previous layer)
    if constexpr (FUSED) {
        if (threadIdx.x == 0) dead = timed_out(prm.err) ? 1 : 0;
        __syncthreads();
    }
    if (!dead) {
    // warp 0 resolves the owners and releases the producer and publisher
    // (barrier 1) while the other consumers stage x; the consumers meet at
    // barrier 4 before computing.  One-call layer: all consumers first route
    // (and stage x), and a CTA whose routing gave up has no owners.
    bool routed = true;
    if constexpr (FUSED)
        if (warp < kConsumerWarps)
            routed = route_phase<NSLOT>(prm, sh, xs, stages, &wbar, rows_issued, queue + 1);
    if (warp == 0) {
        if (routed) {
            resolve_owners(prm, sh, first, blockIdx.x == 0, FUSED ? sh.sids : nullptr);
        } else if (lane == 0) {
            sh.n_owners = 0;
        }
        __syncwarp();
        asm volatile("bar.arrive 1, 96;" ::: "memory");
        asm volatile("bar.sync 4, %0;" ::"n"(kConsumers) : "memory");
    } else if (warp < kConsumerWarps) {
        if constexpr (!FUSED) stage_x_frag<NSLOT>(prm.x, prm.T, D, xs, prm.err, 32, kConsumers - 32);
        asm volatile("bar.sync 4, %0;" ::"n"(kConsumers) : "memory");
    } else {
        asm volatile("bar.sync 1, 96;" ::: "memory");
    }
    pdl_launch_dependents();
    const int n_g = sh.n_owners * nfb, n_all = n_g + sh.n_owners * nrb;
    auto stopped = [&]() { return timed_out(prm.err) || *reinterpret_cast<volatile int*>(&sh.abort) != 0; };
    if (warp == kPublisherWarp) {
        // publisher: release each finished gate|up item to the other CTAs (one
        // gpu-scope fence per batch, then relaxed adds to the owners' counters)
        if (lane == 0) {
            uint32_t tail = 0;
            uint64_t t0 = globaltimer_ns();
            for (bool more = true; more;) {
                // every item queued so far (up to 8), then one fence for the batch
                int v[8];
                int nb = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    v[q] = 0;
                    if (nb == q) {
                        v[q] = (int)ld_acquire_cta(reinterpret_cast<uint32_t*>(&sh.pubq[(tail + q) % kPubRing]));
                        if (v[q] != 0) ++nb;
                    }
                }
                if (nb) {
                    fence_acq_rel_gpu();
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (q < nb) {
                            if (v[q] > 0) red_relaxed_add(done + (v[q] - 1), 1u);
                            else more = false;                  // the end marker
                            st_release_cta(reinterpret_cast<uint32_t*>(&sh.pubq[(tail + q) % kPubRing]), 0u);
                        }
                    }
                    tail += nb;
                    t0 = globaltimer_ns();
                } else {
                    if (globaltimer_ns() - t0 > kWaitLimitNs) { atomicOr(prm.err, kErrTimeout); break; }
                    __nanosleep(32);
                }
            }
        }
    } else if (warp == kProducerWarp) {
        // producer (lane 0): take items from the queue, wait for free stages,
        // issue the copies
        int j = 0, issued = 0;
        bool ok = true;
        // the next item is taken from the queue one step ahead, so the
        // atomic's round trip overlaps the wait for a free stage
        // the next item is taken from the queue one step ahead, so the
        // atomic's round trip overlaps the wait for a free stage
        int next = 0;
        if (lane == 0) next = (int)atomicAdd(queue, 1u);
        for (;; ++j) {
            const int s = j % NS;
            int idx = next, go = 1;
            if (lane == 0) {
                if (idx < n_all) next = (int)atomicAdd(queue, 1u);
                if (j >= NS && !mbar_wait(&sh.empty[s], ((j / NS) - 1) & 1, prm.err)) go = 0;
                else if (stopped()) go = 0;
            }
            go = __shfl_sync(0xffffffffu, go, 0);
            idx = __shfl_sync(0xffffffffu, idx, 0);
            if (!go) { ok = false; break; }
            uint8_t* dst = stages + (size_t)s * stage_bytes;
            if (idx >= n_all) {                       // no more work: tell this stage's team
                if (lane == 0) {
                    sh.stage_item[s] = -1;
                    mbar_arrive(&sh.full[s]);
                }
                ++j;
                break;
            }
            if (idx < n_g) {
                const ItemPos ip = item_pos(idx, nfb, rf);
                const int slot = sh.owners[ip.u].slot;
                if (lane == 0) {
                    sh.stage_item[s] = idx;
                    mbar_arrive_expect_tx(&sh.full[s], 2 * RD.bytes(rf));
                    issue_rows<FMT>(&prm.tm_gu_c, &prm.tm_gu_m, planes_of<FMT>(prm.P, slot, 0), ip.row0, ip.row0, slot,
                                    rf, RD, dst, &sh.full[s]);
                    issue_rows<FMT>(&prm.tm_gu_c, &prm.tm_gu_m, planes_of<FMT>(prm.P, slot, 1), F + ip.row0, ip.row0,
                                    slot, rf, RD, dst + RD.region(rf), &sh.full[s]);
                }
            } else {
                const ItemPos ip = item_pos(idx - n_g, nrb, rd);
                int fine = 1;
                if (lane == 0) {
                    const int slot = sh.owners[ip.u].slot;
                    sh.stage_item[s] = idx;
                    mbar_arrive_expect_tx(&sh.full[s], dn_bytes + hbytes);
                    issue_rows<FMT>(&prm.tm_dn_c, &prm.tm_dn_m, planes_of<FMT>(prm.P, slot, 2), ip.row0, ip.row0, slot,
                                    rd, RF, dst, &sh.full[s]);
                    // the owner's h, once every gate|up item of the owner is published
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire(done + ip.u) < (uint32_t)nfb) {
                        if (timed_out(prm.err) || globaltimer_ns() - t0 > kWaitLimitNs) {
                            atomicOr(prm.err, kErrTimeout);
                            fine = 0;
                            break;
                        }
                        __nanosleep(64);
                    }
                    // (after a give-up the copy still completes the stage's byte count)
                    asm volatile("fence.proxy.async.global;" ::: "memory");   // h was written through the generic proxy
                    bulk_g2s(dst + dn_bytes, prm.hfrag + (size_t)ip.u * F * NSLOT, hbytes, &sh.full[s]);
                }
                ok = __shfl_sync(0xffffffffu, fine, 0) != 0;
            }
            issued = j + 1;
            if (!ok) break;
        }
        if (lane == 0) {
            // the other team's next stage also learns that the work is over
            if (ok) {
                const int s = j % NS;
                if (j < NS || mbar_wait(&sh.empty[s], ((j / NS) - 1) & 1, prm.err)) {
                    sh.stage_item[s] = -1;
                    mbar_arrive(&sh.full[s]);
                }
            } else {
                sh.abort = 1;
            }
            // after a give-up, every issued copy lands before the CTA exits (on the
            // normal path the consumers wait for each staged item themselves)
            if (!ok)
                for (int q = issued - NS; q < issued; ++q)
                    if (q >= 0) mbar_drain(&sh.full[q % NS], (q / NS) & 1);
        }
        __syncwarp();
        if (lane == 0 && atomicAdd(&sh.finished, 1u) == kConsumerWarps) pub_push(sh, kPubEnd);   // the last worker warp
    } else {
        // consumer teams: team tm takes stages j = tm, tm + 2, ... of the ring;
        // the warps of a team work through the same items without waiting on
        // each other (the last one to finish a gate|up item reduces it)
        const int team = warp / kTeamWarps, wt = warp % kTeamWarps;
        float* redt = red + (size_t)team * red_team;
        uint32_t n_gu = 0;                       // gate|up items this team has seen (same order in every warp)
        for (int j = team;; j += kTeams) {
            const int s = j % NS;
            if (!mbar_wait(&sh.full[s], (j / NS) & 1, prm.err)) { if (lane == 0) sh.abort = 1; break; }
            const int idx = sh.stage_item[s];
            if (idx < 0) break;
            const uint8_t* st = stages + (size_t)s * stage_bytes;
            if (idx < n_g) {
                const ItemPos ip = item_pos(idx, nfb, rf);
                const int b = (int)(n_gu % kRedBufs);
                const uint32_t use = n_gu / kRedBufs;     // earlier reductions of buffer b
                ++n_gu;
                float* redb = redt + (size_t)b * (kTeamWarps * red_floats<NSLOT>());
                // buffer b is free once its previous reduction is done (rarely waits)
                bool ok = true;
                if (lane == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_cta(&sh.red_gen[team][b]) < use) {
                        if (stopped() || globaltimer_ns() - t0 > kWaitLimitNs) {
                            atomicOr(prm.err, kErrTimeout);
                            ok = false;
                            break;
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (rf == 16) gateup_partial<FMT, 2, NSLOT>(prm, rf, st, xs, wt, redb + wt * red_floats<NSLOT>());
                else gateup_partial<FMT, 1, NSLOT>(prm, rf, st, xs, wt, redb + wt * red_floats<NSLOT>());
                __syncwarp();
                uint32_t prev = 0;
                if (lane == 0) {
                    mbar_arrive(&sh.empty[s]);
                    asm volatile("atom.acq_rel.cta.shared.add.u32 %0, [%1], 1;"
                                 : "=r"(prev)
                                 : "r"((uint32_t)__cvta_generic_to_shared(&sh.red_cnt[team][b]))
                                 : "memory");
                }
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == kTeamWarps - 1) {            // the last warp of the item reduces it
                    __syncwarp();                        // (orders the other warps' partials, seen by lane 0)
                    gateup_reduce<NSLOT>(prm, ip.u, ip.row0, rf, redb);
                    __syncwarp();
                    if (lane == 0) {
                        sh.red_cnt[team][b] = 0;
                        st_release_cta(&sh.red_gen[team][b], use + 1);
                        pub_push(sh, (uint32_t)(ip.u + 1));
                    }
                }
            } else {
                const ItemPos ip = item_pos(idx - n_g, nrb, rd);
                down_item<FMT, NSLOT>(prm, sh.owners[ip.u], ip.row0, rd, st, st + dn_bytes, wt);
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.empty[s]);
            }
        }
        // the last worker warp to finish tells the publisher that no more items come
        __syncwarp();
        if (lane == 0 && atomicAdd(&sh.finished, 1u) == kConsumerWarps) pub_push(sh, kPubEnd);
    }
    }   // !dead
    if constexpr (FUSED) {
        if (dead && rows_issued && threadIdx.x == 0) mbar_drain(&wbar, 0);   // the Wr copy lands before exit
        // one-call layer: once every CTA's expert rows are written (a grid-wide
        // barrier: release, this CTA's rows; acquire, every other CTA's), each
        // CTA combines its slice of the outputs
        __syncthreads();
        __shared__ int comb_ok;
        if (threadIdx.x == 0) {
            const bool arrived = grid_arrive_wait(queue + 2, prm.err);
            comb_ok = arrived && !dead && sh.n_owners > 0 && !timed_out(prm.err);
        }
        __syncthreads();
        if (comb_ok) combine_slice(prm, sh);
    }
    // last CTA out resets the per-owner counters and the queue for the next call
    // (acq_rel ticket: this CTA's counter updates, ordered before it by the
    // barrier, precede the reset; the last CTA sees every other CTA's)
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t ticket;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(ticket) : "l"(done + kMaxPairs) : "memory");
        if (ticket == gridDim.x - 1) {
            for (int u = 0; u < kMaxPairs; ++u) done[u] = 0u;
            done[kMaxPairs] = 0u;
            done[kMaxPairs + 1] = 0u;
            if constexpr (FUSED) {
                done[kMaxPairs + 2] = 0u;                       // the routing barrier
                done[kMaxPairs + 3] = 0u;                       // the combine barrier
            }
        }
    }
}

template <int FMT, int NSLOT>
size_t smem_for(int D, int F, int rf, int rd, int ns) {
    const size_t fixed = (size_t)D * NSLOT * 2 + kTeams * (size_t)kRedBufs * kTeamWarps * red_floats<NSLOT>() * 4;
    return 128 + fixed + (size_t)ns * stage_size<FMT, NSLOT>(D, F, rf, rd);
}

// Dynamic shared memory available to decode_ffn_kernel<FMT, NSLOT> on the
// current device: the opt-in per-block limit less the kernel's static shared
// memory, capped at kSmemBudget (looked up once per device; 0 if the query fails).
template <int FMT, int NSLOT, bool FUSED>
int smem_budget() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) {
        const int v = cache[dev].load(std::memory_order_relaxed);
        if (v) return v;
    }
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, decode_ffn_kernel<FMT, NSLOT, FUSED>) != cudaSuccess)
        return 0;
    int b = optin - (int)fa.sharedSizeBytes;
    if (b > kSmemBudget) b = kSmemBudget;
    if (dev >= 0 && dev < 64) cache[dev].store(b, std::memory_order_relaxed);
    return b;
}

template <int FMT, int NSLOT, bool FUSED>
moe_status launch_fmt(DecodeParams prm, cudaStream_t s) {
    const PoolView& P = prm.P;
    const int D = P.D, F = P.F;
    const int budget = smem_budget<FMT, NSLOT, FUSED>();
    if (budget <= 0) return MOE_ERR_CUDA;
    // gate|up items of rf features (two 16-row tiles), down items of rd rows
    // (eight 16-row tiles, one per warp of a team), up to 4 stages (3-4 items in
    // flight per SM cover the copy latency)
    int rf = 16, rd = 128;
    while (rf > 8 && smem_for<FMT, NSLOT>(D, F, rf, rd, 2) > (size_t)budget) rf /= 2;
    while (rd > 16 && (size_t)Rows<FMT>::of(F).bytes(rd) > 2 * (size_t)Rows<FMT>::of(D).region(rf)) rd /= 2;
    while (rd > 16 && smem_for<FMT, NSLOT>(D, F, rf, rd, 2) > (size_t)budget) rd /= 2;
    int ns = 4;
    while (ns > 2 && smem_for<FMT, NSLOT>(D, F, rf, rd, ns) > (size_t)budget) --ns;
    prm.rf = rf;
    prm.rd = rd;
    prm.ns = ns;
    const size_t smem = smem_for<FMT, NSLOT>(D, F, rf, rd, ns);
    if (smem > (size_t)budget || F % rf || D % rd) return MOE_ERR_UNSUPPORTED;
    // every bulk copy must be a multiple of 16 bytes
    auto ok16 = [](int K, int n) {
        return ((size_t)Geo<FMT>::code_row(K) * n) % 16 == 0 && ((size_t)Geo<FMT>::meta_row(K) * n) % 16 == 0 &&
               ((size_t)Geo<FMT>::d_row(K) * n) % 16 == 0;
    };
    if (!ok16(D, rf) || !ok16(F, rd)) return MOE_ERR_UNSUPPORTED;
    // tensor maps over every slot: gate|up as 2F rows of D weights, down as D
    // rows of F weights (after the gate and up matrices of the slot)
    const Rows<FMT> RD = Rows<FMT>::of(D), RF = Rows<FMT>::of(F);
    const uint8_t* dn_codes = P.codes + 2 * (size_t)F * RD.cr;
    const uint64_t slots = (uint64_t)P.n_slots;
    if (!padded_rows_map(&prm.tm_gu_c, P.codes, RD.cr, 2 * (uint64_t)F, slots, P.stride_c, RD.c, (uint32_t)rf) ||
        !padded_rows_map(&prm.tm_dn_c, dn_codes, RF.cr, (uint64_t)D, slots, P.stride_c, RF.c, (uint32_t)rd))
        return MOE_ERR_UNSUPPORTED;
    if constexpr (FMT != MOE_Q3_S256) {
        const uint8_t* dn_scales = P.scales + 2 * (size_t)F * RD.mr;
        if (!padded_rows_map(&prm.tm_gu_m, P.scales, RD.mr, 2 * (uint64_t)F, slots, P.stride_s, RD.m, (uint32_t)rf) ||
            !padded_rows_map(&prm.tm_dn_m, dn_scales, RF.mr, (uint64_t)D, slots, P.stride_s, RF.m, (uint32_t)rd))
            return MOE_ERR_UNSUPPORTED;
    } else {
        prm.tm_gu_m = prm.tm_gu_c;
        prm.tm_dn_m = prm.tm_dn_c;
    }
    static std::atomic<uint64_t> attr_done{0};
    if (!once_per_device(attr_done, [] {
            return cudaFuncSetAttribute(decode_ffn_kernel<FMT, NSLOT, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        smem_budget<FMT, NSLOT, FUSED>()) == cudaSuccess;
        }))
        return MOE_ERR_CUDA;
    if constexpr (FUSED) {
        // routing in the kernel: x (bf16) fits in the stage ring, one logit warp per expert
        prm.route_j = (prm.E + device_sm_count() - 1) / device_sm_count();
        const size_t ring = (size_t)ns * stage_size<FMT, NSLOT>(D, F, rf, rd);
        if ((size_t)prm.T * D * 2 > ring || prm.route_j > kConsumerWarps) return MOE_ERR_UNSUPPORTED;
        prm.route_wr_smem = wr_ring_offset(prm.T, D) + (size_t)prm.route_j * D * 2 <= ring ? 1 : 0;
    }
    // the one-call layer's CTAs meet at grid-wide barriers: a cooperative launch
    cudaError_t e = launch_pdl_ex(FUSED, decode_ffn_kernel<FMT, NSLOT, FUSED>, dim3(device_sm_count()), dim3(kThreads),
                                  smem, s, prm);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

// ws layout: [0,4) reserved, [4,8) device error word, [64, 64 + 4*(kMaxPairs+1))
// completion counters (zero before the first call; every completed call leaves
// them zero), [1024, ...) h of every owner (fp16, fragment order, 4 token
// columns for T <= 4, else 8).
size_t decode_workspace_bytes(int T, int D, int F, int k) {
    (void)D; (void)k;
    return 1024 + (size_t)kMaxPairs * (T <= 4 ? 4 : 8) * F * sizeof(uint16_t);
}

namespace {
// tokens [t0, t0 + T) of a batch of T_all tokens whose expert_out layout is
// rowmap [T_all][k+1], then fp32 rows [T_all * (k+1)][D]
DecodeParams expert_params(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x, int T,
                           const int32_t* ids, int k, void* expert_out, int32_t* miss_list, int32_t* miss_count,
                           int T_all = 0, int t0 = 0) {
    if (T_all == 0) T_all = T;
    DecodeParams prm{};
    prm.P = P;
    prm.slot_table = slot_table;
    prm.E = E;
    prm.x = x;
    prm.T = T;
    prm.ids = ids;
    prm.k = k;
    prm.rowmap = reinterpret_cast<int32_t*>(expert_out) + (size_t)t0 * (k + 1);
    prm.yrows = reinterpret_cast<float*>(reinterpret_cast<char*>(expert_out) + rowmap_bytes(T_all, k)) +
                (size_t)t0 * (k + 1) * P.D;
    prm.miss_list = miss_list;
    prm.miss_count = miss_count;
    prm.t0 = t0;
    prm.miss_append = t0 > 0 ? 1 : 0;
    return prm;
}

template <bool FUSED>
moe_status launch_any(DecodeParams prm, cudaStream_t s) {
    if (prm.T <= 4) {
        switch (prm.P.fmt) {
            case MOE_Q2_32: return launch_fmt<MOE_Q2_32, 4, FUSED>(prm, s);
            case MOE_Q3_32: return launch_fmt<MOE_Q3_32, 4, FUSED>(prm, s);
            default: return launch_fmt<MOE_Q3_S256, 4, FUSED>(prm, s);
        }
    }
    switch (prm.P.fmt) {
        case MOE_Q2_32: return launch_fmt<MOE_Q2_32, 8, FUSED>(prm, s);
        case MOE_Q3_32: return launch_fmt<MOE_Q3_32, 8, FUSED>(prm, s);
        default: return launch_fmt<MOE_Q3_S256, 8, FUSED>(prm, s);
    }
}

// one-call layer ws: [4,8) error word, [64, ...) counters (as the expert
// pass's, plus the routing and combine barriers), [1024, 33792) logits [T][E]
// fp32, then h.
constexpr size_t kLayerLogits = 1024, kLayerH = 1024 + (size_t)kDecodeMaxT * 1024 * 4;
}  // namespace

moe_status launch_decode_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x, int T,
                                 const int32_t* ids, int k, void* expert_out, int32_t* miss_list,
                                 int32_t* miss_count, void* ws, cudaStream_t s) {
    if (P.D % kUnitK || P.F % kUnitK || T > kDecodeLayoutMaxT) return MOE_ERR_UNSUPPORTED;
    // up to 8 tokens per launch, in token order (each later launch appends its misses
    // and writes its rows after the earlier ones')
    for (int t0 = 0; t0 < T; t0 += kDecodeMaxT) {
        const int n = T - t0 < kDecodeMaxT ? T - t0 : kDecodeMaxT;
        DecodeParams prm = expert_params(P, slot_table, E, x + (size_t)t0 * P.D, n, ids + (size_t)t0 * k, k,
                                         expert_out, miss_list, miss_count, T, t0);
        prm.err = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 4);
        prm.done = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 64);
        prm.hfrag = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(ws) + 1024);
        const moe_status st = launch_any<false>(prm, s);
        if (st != MOE_OK) return st;
    }
    return MOE_OK;
}

size_t layer_workspace_bytes(int T, int D, int F, int E, int k) {
    (void)D; (void)E; (void)k;
    return kLayerH + (size_t)kMaxPairs * (T <= 4 ? 4 : 8) * F * sizeof(uint16_t);
}

moe_status launch_layer_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x, int T,
                                const uint16_t* Wr, const float* bias, int k, int32_t* ids, float* gates,
                                void* expert_out, int32_t* miss_list, int32_t* miss_count, const uint16_t* residual,
                                uint16_t* out, void* ws, cudaStream_t s) {
    if (P.D % kUnitK || P.F % kUnitK || T > kDecodeMaxT || E > 1024) return MOE_ERR_UNSUPPORTED;
    char* w = reinterpret_cast<char*>(ws);
    DecodeParams prm = expert_params(P, slot_table, E, x, T, nullptr, k, expert_out, miss_list, miss_count);
    prm.err = reinterpret_cast<uint32_t*>(w + 4);
    prm.done = reinterpret_cast<uint32_t*>(w + 64);
    prm.logits = reinterpret_cast<float*>(w + kLayerLogits);
    prm.hfrag = reinterpret_cast<uint16_t*>(w + kLayerH);
    prm.Wr = Wr;
    prm.bias = bias;
    prm.ids_out = ids;
    prm.gates_out = gates;
    prm.residual = residual;
    prm.out = out;
    return launch_any<true>(prm, s);
}

}  // namespace moe
