// route.cu — router logits in the canonical fp32 order, top-k and gates.
//
// Routing runs on the GPU (greenbean-ai "Strata 如何讓 12GB 顯卡跑
// Qwen3.8-Flash-Next", §二); top-10 of 512 experts per token per layer
// (wiselychen RTX 5090 report, "30 秒定位").  The canonical order (32 lane
// partial sums of fmaf over elements 256c + 8L + j, pairwise xor-butterfly,
// then + bias) is what makes the selected ids reproducible bit for bit.
#include "common.cuh"
#include "kernels.cuh"
#include "once.cuh"
#include "route_warp.cuh"
#include "sync.cuh"

namespace moe {

// Decode route (T <= 8, x staged in shared memory): one warp per expert
// computes its logits for all T
// tokens, then the last block to finish selects every token's top-k.  The
// block counter lives in ws and wraps back to zero on every completed launch.
// Wr is not produced by the preceding kernel: one bulk copy brings the block's
// four expert rows into shared memory, and each warp loads its expert's bias,
// before waiting on the producer of x.
// x is staged once per block as fp32 in shared memory.
template <int NT>
__global__ void __launch_bounds__(128) route_decode_kernel(const uint16_t* __restrict__ x, int T, int D,
                                                           const uint16_t* __restrict__ Wr,
                                                           const float* __restrict__ bias, int E, int k,
                                                           float* __restrict__ logits, int32_t* __restrict__ ids,
                                                           float* __restrict__ gates, unsigned int* counter,
                                                           uint32_t* err) {
    extern __shared__ __align__(128) uint8_t rsm[];
    float* xsf = reinterpret_cast<float*>(rsm);                                // [T][D], canon_stage_pos order
    uint16_t* wsm = reinterpret_cast<uint16_t*>(rsm + (size_t)T * D * 4);      // the block's Wr rows [4][D]
    __shared__ uint64_t wbar;
    const int warp = threadIdx.x >> 5;
    const int e0 = blockIdx.x * 4, e = e0 + warp;
    if (threadIdx.x == 0) {
        mbar_init(&wbar, 1);
        fence_mbar_init();
        const uint32_t bytes = (uint32_t)min(4, E - e0) * (uint32_t)D * 2u;
        mbar_arrive_expect_tx(&wbar, bytes);
        bulk_g2s(wsm, Wr + (size_t)e0 * D, bytes, &wbar);
    }
    const float bias_e = (bias && e < E) ? __ldg(bias + e) : 0.0f;   // a weight too: load it now
    pdl_wait();
    stage_x_canon(x, T, D, xsf, (int)threadIdx.x, 128);
    __syncthreads();
    pdl_launch_dependents();
    const bool have_w = mbar_wait(&wbar, 0, err);
    if (!have_w && threadIdx.x == 0) mbar_drain(&wbar, 0);   // the copy lands before the CTA moves on
    if (e < E && have_w) canon_logits_warp_staged<NT>(xsf, T, D, wsm + (size_t)warp * D, bias != nullptr, bias_e, E, e, logits);
    // the last block to arrive selects: one acq_rel ticket per block (release:
    // the block's logits, ordered before it by the barrier; acquire: every
    // other block's logits for the last one)
    __shared__ bool last;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int prev;
        asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;" : "=r"(prev) : "l"(counter), "r"(gridDim.x - 1) : "memory");
        last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!last) return;
    if (timed_out(err)) {            // some block gave up: no selection from incomplete logits
        for (int i = threadIdx.x; i < T * k; i += blockDim.x) { ids[i] = -1; gates[i] = 0.f; }
        return;
    }
    for (int t = warp; t < T; t += 4) topk_warp(logits + (size_t)t * E, E, k, ids + (size_t)t * k, gates + (size_t)t * k);
}

moe_status launch_route(const uint16_t* x, int T, int D, const uint16_t* Wr, const float* bias, int E,
                        int k, int32_t* ids, float* gates, float* logits, void* ws, cudaStream_t s) {
    unsigned int* counter = reinterpret_cast<unsigned int*>(ws);
    uint32_t* rerr = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 4);
    float* lg = logits ? logits : reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + 256);
    cudaError_t e;
    // decode router: up to 8 tokens per launch, as many launches as the decode
    // expert pass takes (each launch stages its tokens' x as fp32 and four router
    // rows in shared memory)
    const int tc = T < kRouteDecodeMaxT ? T : kRouteDecodeMaxT;
    if (T <= kDecodeLayoutMaxT && (size_t)(4 * tc + 8) * D <= kRouteDecodeSmem) {
        const dim3 grid((E + 3) / 4), block(128);
        static std::atomic<uint64_t> attr{0};
        if (!once_per_device(attr, [] {
                const int b = (int)kRouteDecodeSmem;
                return cudaFuncSetAttribute(route_decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess &&
                       cudaFuncSetAttribute(route_decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess &&
                       cudaFuncSetAttribute(route_decode_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess &&
                       cudaFuncSetAttribute(route_decode_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess &&
                       cudaFuncSetAttribute(route_decode_kernel<5>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess &&
                       cudaFuncSetAttribute(route_decode_kernel<6>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess &&
                       cudaFuncSetAttribute(route_decode_kernel<7>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess &&
                       cudaFuncSetAttribute(route_decode_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) == cudaSuccess;
            }))
            return MOE_ERR_CUDA;
        for (int t0 = 0; t0 < T; t0 += kRouteDecodeMaxT) {
            const int n = T - t0 < kRouteDecodeMaxT ? T - t0 : kRouteDecodeMaxT;
            const size_t smem = (size_t)n * D * sizeof(float) + (size_t)4 * D * sizeof(uint16_t);
            const uint16_t* xc = x + (size_t)t0 * D;
            float* lc = lg + (size_t)t0 * E;
            int32_t* ic = ids + (size_t)t0 * k;
            float* gc = gates + (size_t)t0 * k;
            switch (n) {
                case 1: e = launch_pdl(route_decode_kernel<1>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
                case 2: e = launch_pdl(route_decode_kernel<2>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
                case 3: e = launch_pdl(route_decode_kernel<3>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
                case 4: e = launch_pdl(route_decode_kernel<4>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
                case 5: e = launch_pdl(route_decode_kernel<5>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
                case 6: e = launch_pdl(route_decode_kernel<6>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
                case 7: e = launch_pdl(route_decode_kernel<7>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
                default: e = launch_pdl(route_decode_kernel<8>, grid, block, smem, s, xc, n, D, Wr, bias, E, k, lc, ic, gc, counter, rerr); break;
            }
            if (e != cudaSuccess) return MOE_ERR_CUDA;
        }
        return MOE_OK;
    }
    // prefill: tensor-core logits, then canonical logits of each token's candidates
    float* wnorm = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + 256 +
                                            ((size_t)T * E * sizeof(float) + 255) / 256 * 256);
    uint32_t* err = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 4);
    return launch_route_prefill(x, T, D, Wr, bias, E, k, ids, gates, lg, wnorm, err, s);
}

// ws: [0,4) decode block counter, [4,8) device error word, [256, ...) logits
// scratch [T][E] fp32 (used when the caller passes no logits buffer), then the
// expert norms of the prefill router.
size_t route_workspace_bytes(int T, int D, int E, int k) {
    (void)D; (void)k;
    return 256 + ((size_t)T * E * sizeof(float) + 255) / 256 * 256 + ((size_t)E * sizeof(float) + 255) / 256 * 256;
}

}  // namespace moe

// ---------------------------------------------------------------- no-allocation entry point
// Scratch for moe_route_topk_static: a 256-byte header (word 0 = the block
// counter of the last-block top-k, word 1 = the device error word) followed by room for the logits of up to
// kStaticMaxT tokens x kStaticMaxE experts.  Every GPU that loads this library
// holds it until the process exits.
namespace {
constexpr int kStaticMaxT = 4;
constexpr int kStaticMaxE = 1024;
constexpr size_t kStaticScratchBytes = 256 + (size_t)kStaticMaxT * kStaticMaxE * sizeof(float);
static __device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];
constexpr int kMaxDevices = 64;
static void* g_scratch_ptr[kMaxDevices];
}  // namespace

extern "C" moe_status moe_route_topk_static(const uint16_t* x, int T, int D, const uint16_t* Wr,
                                             const float* bias, int E, int k, int32_t* ids, float* gates,
                                             float* logits, moe_stream_t stream) {
    if (T < 0 || D <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (D % 256 || D > 8192 || k > moe::kMaxTopK || E < k) return MOE_ERR_UNSUPPORTED;
    if (T > kStaticMaxT || E > kStaticMaxE) return MOE_ERR_UNSUPPORTED;   // beyond the static scratch
    if (T == 0) return MOE_OK;
    if (!x || !Wr || !ids || !gates) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)x % 16) || ((uintptr_t)Wr % 16) || (logits && ((uintptr_t)logits % 16))) return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    if (!g_scratch_ptr[dev]) {
        // host code only holds a stand-in for the array: ask the runtime for the
        // device address once per device, with that device current
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    void* ws = g_scratch_ptr[dev];
    cudaStream_t s = (cudaStream_t)stream;
    // the block counter and the device error word start at zero on every call
    // (a call that did not complete may have left either set)
    if (cudaMemsetAsync(ws, 0, 2 * sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    return moe::launch_route(x, T, D, Wr, bias, E, k, ids, gates, logits, ws, s);
}

