// route_tc.cu — prefill router (T > 4): logits of all T x E pairs on the
// tensor cores, then a canonical-order recomputation of every expert that can
// reach a token's top-k, so the ids and gates are those of the canonical
// logits (route.cu) bit for bit.
//
// Routing runs on the GPU (greenbean-ai "Strata 如何讓 12GB 顯卡跑
// Qwen3.8-Flash-Next", §二); top-10 of 512 experts per token (wiselychen RTX
// 5090 report, "30 秒定位").
//
// Error bound.  Both the tensor-core logit l~ (bf16 products, exact in fp32,
// accumulated in fp32 over D/16 MMA steps) and the canonical one l (32 chains
// of D/32 fmaf, then 5 pairwise adds) are sums of the same exact products, so
// |l~ - l| <= (D/16 + D/32 + 64) 2^-23 sum_i |x_i w_i| <= 2^-12 |x|_2 |w|_2
// for D <= 8192.  Every expert whose l~ lies within 2 M = 2^-11 |x|_2 max|w|_2
// of the k-th largest l~ is a candidate: the canonical top-k is among them
// (any other expert has l < l~_k - M <= l of each of the k best candidates).
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tmap.cuh"
#include "once.cuh"
#include "route_warp.cuh"
#include "sync.cuh"

namespace moe {
namespace {

constexpr int kRM = 128;          // tokens per tile (MMA M)
constexpr int kRN = 128;          // experts per tile (MMA N)
constexpr int kRK = 64;           // K per stage: one 128-byte swizzle atom of bf16
constexpr int kRStages = 4;
constexpr uint32_t kRStageBytes = (kRM + kRN) * kRK * 2;
constexpr int kRThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

MOE_DEVINL uint64_t r_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3ffffu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// kind::f16 with A = B = bf16, D = f32, both K-major, M = 128, N = kRN.
constexpr uint32_t kRIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kRN >> 3) << 17) | ((uint32_t)(kRM >> 4) << 24);

MOE_DEVINL void r_tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Logits of a 128-token x 128-expert tile: TMA streams x and Wr tiles, one
// thread issues tcgen05 MMAs into a TMEM accumulator, four warps add the bias
// and store fp32 rows.
__global__ void __launch_bounds__(kRThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                     const float* __restrict__ bias, int T, int D, int E, float* __restrict__ logits, uint32_t* err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full[kRStages], empty[kRStages], done;
    __shared__ uint32_t tmem_base;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = blockIdx.x * kRN, t0 = blockIdx.y * kRM;
    const int KT = D / kRK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(&done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"((uint32_t)kRN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base;
    pdl_wait();
    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < KT; ++j) {
                const int s = j % kRStages;
                if (j >= kRStages && !mbar_wait(&empty[s], ((j / kRStages) - 1) & 1, err)) break;
                uint8_t* st = smem + s * kRStageBytes;
                mbar_arrive_expect_tx(&full[s], kRStageBytes);
                r_tma_2d(smem_u32(st), &map_x, j * kRK, t0, &full[s]);
                r_tma_2d(smem_u32(st + kRM * kRK * 2), &map_w, j * kRK, e0, &full[s]);
                issued = j + 1;
            }
            for (int j = issued - kRStages; j < issued; ++j)
                if (j >= 0) mbar_drain(&full[j % kRStages], (j / kRStages) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            bool issued = false;
            for (int j = 0; j < KT; ++j) {
                const int s = j % kRStages;
                if (!mbar_wait(&full[s], (j / kRStages) & 1, err)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t a = smem_u32(smem + s * kRStageBytes), b = a + kRM * kRK * 2;
#pragma unroll
                for (int kk = 0; kk < kRK / 16; ++kk) {
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                        "l"(r_desc_sw128(a + kk * 32)), "l"(r_desc_sw128(b + kk * 32)), "r"(kRIdesc), "r"(acc));
                }
                issued = true;
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&empty[s]))
                             : "memory");
            }
            if (issued)
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&done))
                             : "memory");
            mbar_drain(&done, 0);
        }
        __syncwarp();
    } else {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. (tokens of the tile)
        const int q = warp & 3;
        const int t = t0 + 32 * q + lane;
        if (mbar_wait(&done, 0, err)) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            for (int c = 0; c < kRN; c += 16) {
                uint32_t v[16];
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                      "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                    : "r"(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (t < T) {
                    float o[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int e = e0 + c + i;
                        o[i] = __uint_as_float(v[i]) + ((bias && e < E) ? __ldg(bias + e) : 0.f);
                    }
                    float* dst = logits + (size_t)t * E + e0 + c;
                    if ((E & 3) == 0 && e0 + c + 16 <= E) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (e0 + c + i < E) dst[i] = o[i];
                    }
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kRN) : "memory");
    }
}

// |Wr_e|_2 for every expert (one warp per expert).
__global__ void __launch_bounds__(256) wnorm_kernel(const uint16_t* __restrict__ Wr, int D, int E, float* __restrict__ wn) {
    const int e = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    pdl_wait();   // wn may still be read by the previous call's selection
    if (e >= E) return;
    float s = 0.f;
    for (int i = 8 * lane; i < D; i += 256) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(Wr + (size_t)e * D + i));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float a = bf16lo(ww[h]), b = bf16hi(ww[h]);
            s = __fmaf_rn(a, a, __fmaf_rn(b, b, s));
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) wn[e] = sqrtf(s) * 1.0001f;   // rounded up: used as an upper bound
}

constexpr int kSelWarps = 8;
constexpr int kMaxRouterE = 1024;     // the largest expert count the selection takes

// Canonical logits (+ bias) of the n <= NC experts es[0..n) for one token
// (bf16 row xrow): for each expert the order and arithmetic of
// canon_logit_one, with the token row read and unpacked once for all of them
// and the router rows of the next 256-element chunk in flight while the
// current one is summed.  Lane 0 stores expert es[j]'s logit into out[es[j]].
template <int NC>
__device__ __forceinline__ void canon_logits_multi(const uint16_t* __restrict__ xrow, int D,
                                                   const uint16_t* __restrict__ Wr, const float* __restrict__ bias,
                                                   const uint16_t* es, int n, float* out) {
    const int lane = threadIdx.x & 31;
    const uint16_t* wrow[NC];
    float acc[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        wrow[j] = Wr + (size_t)es[j < n ? j : 0] * D + 8 * lane;
        acc[j] = 0.0f;
    }
    const int nc = D >> 8;
    auto load = [&](uint4 (&w)[NC], int c) {
#pragma unroll
        for (int j = 0; j < NC; ++j) w[j] = (j < n && c < nc) ? ld_nc_u128(wrow[j] + 256 * c) : make_uint4(0, 0, 0, 0);
    };
    auto sum = [&](const uint4 (&w)[NC], int c) {
        const uint4 xv4 = *reinterpret_cast<const uint4*>(xrow + 256 * c + 8 * lane);
        const uint32_t xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
        float xf[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) { xf[2 * q] = bf16lo(xv[q]); xf[2 * q + 1] = bf16hi(xv[q]); }
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            if (j < n) {
                const uint32_t wv[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[j] = __fmaf_rn(xf[2 * q], bf16lo(wv[q]), acc[j]);
                    acc[j] = __fmaf_rn(xf[2 * q + 1], bf16hi(wv[q]), acc[j]);
                }
            }
        }
    };
    // two buffers in turn: chunk c is summed while chunk c + 1 is in flight,
    // then its buffer is refilled with chunk c + 2
    uint4 wa[NC], wb[NC];
    load(wa, 0);
    load(wb, 1);
    for (int c = 0; c < nc; c += 2) {
        sum(wa, c);
        load(wa, c + 2);
        if (c + 1 < nc) {
            sum(wb, c + 1);
            load(wb, c + 3);
        }
    }
#pragma unroll
    for (int j = 0; j < NC; ++j) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc[j] = __fadd_rn(acc[j], __shfl_xor_sync(0xffffffffu, acc[j], off));
    }
    if (lane == 0) {
#pragma unroll
        for (int j = 0; j < NC; ++j)
            if (j < n) out[es[j]] = bias ? __fadd_rn(acc[j], __ldg(bias + es[j])) : acc[j];
    }
}

// One warp per token (E <= 32 NV): the k-th largest approximate logit (by the
// warp top-k on the approximate row), the candidates within twice the margin
// below it, their canonical logits (four experts at a time), then the exact
// top-k and gates over the canonical row (every other expert at -inf).
template <int NV>
__global__ void __launch_bounds__(kSelWarps * 32) router_select_kernel(const uint16_t* __restrict__ x, int T, int D,
                                                                       const uint16_t* __restrict__ Wr,
                                                                       const float* __restrict__ bias, int E, int k,
                                                                       const float* __restrict__ approx,
                                                                       const float* __restrict__ wn,
                                                                       int32_t* __restrict__ ids, float* __restrict__ gates,
                                                                       const uint32_t* err) {
    extern __shared__ float rows[];          // [kSelWarps][E] logits, then [kSelWarps][E] candidate ids (16-bit)
    __shared__ int32_t s_kid[kSelWarps][kMaxTopK];
    __shared__ float s_kg[kSelWarps][kMaxTopK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kSelWarps + warp;
    pdl_wait();
    if (t >= T) return;
    if (timed_out(err)) {            // the logits kernel gave up: no selection from incomplete logits
        if (lane < k) { ids[(size_t)t * k + lane] = -1; gates[(size_t)t * k + lane] = 0.f; }
        return;
    }
    float* row = rows + (size_t)warp * E;
    uint16_t* cl = reinterpret_cast<uint16_t*>(rows + (size_t)kSelWarps * E) + (size_t)warp * E;
    const float* ar = approx + (size_t)t * E;
    const uint16_t* xr = x + (size_t)t * D;
    // every load of the approximate row, the expert norms and the first 16
    // chunks of x in flight together
    float av[NV], wv[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        av[i] = e < E ? __ldg(ar + e) : 0.f;
        wv[i] = e < E ? __ldg(wn + e) : 0.f;
    }
    // |x_t|_2 (the same summation order as one chunk at a time) and max_e |Wr_e|_2
    float sx = 0.f, wmax = 0.f;
    constexpr int kXB = 8;
    for (int c0 = 0; c0 < D / 256; c0 += kXB) {
        uint4 v[kXB];
#pragma unroll
        for (int q = 0; q < kXB; ++q)
            v[q] = c0 + q < D / 256 ? __ldg(reinterpret_cast<const uint4*>(xr + 256 * (c0 + q) + 8 * lane))
                                    : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int q = 0; q < kXB; ++q) {
            if (c0 + q < D / 256) {
                const uint32_t vv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float a = bf16lo(vv[h]), b = bf16hi(vv[h]);
                    sx = __fmaf_rn(a, a, __fmaf_rn(b, b, sx));
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        if (lane + 32 * i < E) row[lane + 32 * i] = av[i];
        wmax = fmaxf(wmax, wv[i]);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        sx += __shfl_xor_sync(0xffffffffu, sx, off);
        wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, off));
    }
    const float margin2 = ldexpf(sqrtf(sx) * 1.0001f * wmax, -11);   // 2 M
    __syncwarp();
    // k-th largest approximate logit: the expert the top-k of the approximate row ranks k-th
    topk_warp_n<NV, true>(row, E, k, s_kid[warp], s_kg[warp]);
    __syncwarp();
    const int kid = s_kid[warp][k - 1];
    const float kth = (unsigned)kid < (unsigned)E ? row[kid] : -INFINITY;
    const float thr = kth - margin2;
    __syncwarp();                    // every lane has read row[kid] before the row is reset
    // candidates in ascending expert order; the row is then reset to -inf
    int n = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        const bool cand = e < E && av[i] >= thr;
        const uint32_t m = __ballot_sync(0xffffffffu, cand);
        if (cand) cl[n + __popc(m & ((1u << lane) - 1u))] = (uint16_t)e;
        n += __popc(m);
        if (e < E) row[e] = -INFINITY;
    }
    __syncwarp();
    for (int c0 = 0; c0 < n; c0 += 4) canon_logits_multi<4>(xr, D, Wr, bias, cl + c0, min(4, n - c0), row);
    __syncwarp();
    topk_warp_n<NV, true>(row, E, k, ids + (size_t)t * k, gates + (size_t)t * k);
}

// bf16 [rows][D], boxes of 64 x 128 rows, 128B swizzle
bool bf16_rows_map(CUtensorMap* m, const void* base, int D, int rows) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kRK, 128};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// logits: the T x E approximate logits (caller's buffer or scratch); scratch
// also holds the expert norms after the logits.
moe_status launch_route_prefill(const uint16_t* x, int T, int D, const uint16_t* Wr, const float* bias, int E, int k,
                                int32_t* ids, float* gates, float* logits, float* wnorm, uint32_t* err,
                                cudaStream_t s) {
    CUtensorMap mx, mw;
    if (!bf16_rows_map(&mx, x, D, T) || !bf16_rows_map(&mw, Wr, D, E)) return MOE_ERR_CUDA;
    const size_t smem = kRStages * kRStageBytes + 1024;
    static std::atomic<uint64_t> attr{0};
    if (!once_per_device(attr, [&] {
            return cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
                       cudaSuccess &&
                   cudaFuncSetAttribute(router_select_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)(kSelWarps * 512 * (sizeof(float) + sizeof(uint16_t)))) == cudaSuccess &&
                   cudaFuncSetAttribute(router_select_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)(kSelWarps * kMaxRouterE * (sizeof(float) + sizeof(uint16_t)))) == cudaSuccess;
        }))
        return MOE_ERR_CUDA;
    cudaError_t e = launch_pdl(wnorm_kernel, dim3((E + 7) / 8), dim3(256), 0, s, Wr, D, E, wnorm);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_pdl(router_tc_kernel, dim3((E + kRN - 1) / kRN, (T + kRM - 1) / kRM), dim3(kRThreads), smem, s, mx, mw,
                   bias, T, D, E, logits, err);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const size_t sel_smem = (size_t)kSelWarps * E * (sizeof(float) + sizeof(uint16_t));
    e = launch_pdl(E <= 512 ? router_select_kernel<16> : router_select_kernel<32>, dim3((T + kSelWarps - 1) / kSelWarps), dim3(kSelWarps * 32), sel_smem, s, x,
                   T, D, Wr, bias, E, k, (const float*)logits, (const float*)wnorm, ids, gates, (const uint32_t*)err);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
