// route.cu — router logits in the canonical fp32 order, top-k and gates.
//
// Routing runs on the GPU (greenbean-ai "Strata 如何讓 12GB 顯卡跑
// Qwen3.8-Flash-Next", §二); top-10 of 512 experts per token per layer
// (wiselychen RTX 5090 report, "30 秒定位").  The canonical order (32 lane
// partial sums of fmaf over elements 256c + 8L + j, pairwise xor-butterfly,
// then + bias) is what makes the selected ids reproducible bit for bit.
#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

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

// "a before b": larger logit, then lower id.
__device__ __forceinline__ bool cand_better(float va, int ea, float vb, int eb) {
    return va > vb || (va == vb && ea < eb);
}

// Compare-exchange for a descending order by (value, then lower id).
__device__ __forceinline__ void cex(float& va, int& ea, float& vb, int& eb) {
    if (cand_better(vb, eb, va, ea)) {
        const float tv = va; va = vb; vb = tv;
        const int te = ea; ea = eb; eb = te;
    }
}

// One warp selects the top-k of one token's E logits (E <= 32 * NV) and
// writes ids and gates.  Each lane sorts its NV values once (a bitonic network
// in registers); each of the k rounds then takes the warp's best lane head and
// the winning lane shifts its list.  Gates are formed in double from the
// selected fp32 logits.
template <int NV>
__device__ void topk_warp_n(const float* __restrict__ lrow, int E, int k, int32_t* __restrict__ ids,
                            float* __restrict__ gates) {
    const int lane = threadIdx.x & 31;
    float v[NV];
    int e[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        e[i] = lane + 32 * i;
        v[i] = (e[i] < E) ? __ldcg(lrow + e[i]) : -INFINITY;
        if (e[i] >= E) e[i] = 0x7fffffff;
    }
    // bitonic sort, descending
#pragma unroll
    for (int kk = 2; kk <= NV; kk <<= 1) {
#pragma unroll
        for (int j = kk >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    if ((i & kk) == 0) cex(v[i], e[i], v[l], e[l]);
                    else cex(v[l], e[l], v[i], e[i]);
                }
            }
        }
    }
    float my_v = 0.f, l0 = 0.f;
    int my_e = 0;
    for (int r = 0; r < k; ++r) {
        float wv = v[0];
        int we = e[0];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, wv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, we, off);
            if (cand_better(ov, oe, wv, we)) { wv = ov; we = oe; }
        }
        if (r == 0) l0 = wv;
        if (lane == r) { my_v = wv; my_e = we; }
        if (e[0] == we) {                       // this lane supplied the winner: pop its head
#pragma unroll
            for (int i = 0; i + 1 < NV; ++i) { v[i] = v[i + 1]; e[i] = e[i + 1]; }
            v[NV - 1] = -INFINITY;
            e[NV - 1] = 0x7fffffff;
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

// Decode route (T <= 4): one warp per expert computes its logits for all T
// tokens, then the last block to finish selects every token's top-k.  The
// block counter lives in ws and wraps back to zero on every completed launch.
// Wr rows are prefetched into L2 before waiting on the producer of x.
template <int NT>
__global__ void __launch_bounds__(128) route_decode_kernel(const uint16_t* __restrict__ x, int T, int D,
                                                           const uint16_t* __restrict__ Wr,
                                                           const float* __restrict__ bias, int E, int k,
                                                           float* __restrict__ logits, int32_t* __restrict__ ids,
                                                           float* __restrict__ gates, unsigned int* counter) {
    extern __shared__ __align__(16) uint16_t xsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 4 + warp;
    if (e < E && lane == 0) prefetch_l2(Wr + (size_t)e * D, (uint32_t)D * 2);
    pdl_wait();
    for (int i = threadIdx.x; i < T * D / 8; i += blockDim.x)
        reinterpret_cast<uint4*>(xsm)[i] = __ldg(reinterpret_cast<const uint4*>(x) + i);
    __syncthreads();
    pdl_launch_dependents();
    if (e < E) {
        const uint16_t* xr[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) xr[t] = xsm + (size_t)t * D;
        canon_logits_warp<NT>(xr, T, D, Wr, bias, E, e, logits);
    }
    __shared__ bool last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = (atomicInc(counter, gridDim.x - 1) == gridDim.x - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    if (warp < T) topk_warp(logits + (size_t)warp * E, E, k, ids + (size_t)warp * k, gates + (size_t)warp * k);
}

// Prefill route, canonical path: grid (E/8, T/4).
__global__ void __launch_bounds__(256) route_logits_kernel(const uint16_t* __restrict__ x, int T, int D,
                                                           const uint16_t* __restrict__ Wr,
                                                           const float* __restrict__ bias, int E,
                                                           float* __restrict__ logits) {
    pdl_wait();
    const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int t0 = blockIdx.y * 4;
    if (e < E) {
        const uint16_t* xr[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) xr[t] = x + (size_t)min(t0 + t, T - 1) * D;
        canon_logits_warp<4>(xr, min(4, T - t0), D, Wr, bias, E, e, logits + (size_t)t0 * E);
    }
}

__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int32_t* __restrict__ ids, float* __restrict__ gates) {
    pdl_wait();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t < T) topk_warp(logits + (size_t)t * E, E, k, ids + (size_t)t * k, gates + (size_t)t * k);
}

int route_num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

moe_status launch_route(const uint16_t* x, int T, int D, const uint16_t* Wr, const float* bias, int E,
                        int k, int32_t* ids, float* gates, float* logits, void* ws, cudaStream_t s) {
    unsigned int* counter = reinterpret_cast<unsigned int*>(ws);
    float* lg = logits ? logits : reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + 256);
    cudaError_t e;
    if (T <= kDecodeMaxT) {
        const dim3 grid((E + 3) / 4), block(128);
        const size_t smem = (size_t)T * D * sizeof(uint16_t);
        static bool attr = false;
        if (!attr) {
            cudaFuncSetAttribute(route_decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
            cudaFuncSetAttribute(route_decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
            cudaFuncSetAttribute(route_decode_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
            cudaFuncSetAttribute(route_decode_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
            attr = true;
        }
        switch (T) {
            case 1: e = launch_pdl(route_decode_kernel<1>, grid, block, smem, s, x, T, D, Wr, bias, E, k, lg, ids, gates, counter); break;
            case 2: e = launch_pdl(route_decode_kernel<2>, grid, block, smem, s, x, T, D, Wr, bias, E, k, lg, ids, gates, counter); break;
            case 3: e = launch_pdl(route_decode_kernel<3>, grid, block, smem, s, x, T, D, Wr, bias, E, k, lg, ids, gates, counter); break;
            default: e = launch_pdl(route_decode_kernel<4>, grid, block, smem, s, x, T, D, Wr, bias, E, k, lg, ids, gates, counter); break;
        }
        return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
    (void)route_num_sms;
    e = launch_pdl(route_logits_kernel, dim3((E + 7) / 8, (T + 3) / 4), dim3(256), 0, s, x, T, D, Wr, bias, E, lg);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_pdl(topk_kernel, dim3((T + 7) / 8), dim3(256), 0, s, (const float*)lg, T, E, k, ids, gates);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t route_workspace_bytes(int T, int D, int E, int k) {
    (void)D; (void)k;
    return 256 + (size_t)T * E * sizeof(float);
}

}  // namespace moe

// ---------------------------------------------------------------- no-allocation entry point
// Scratch for moe_route_topk_static: a 256-byte header (word 0 = the block
// counter of the last-block top-k) followed by room for the logits of up to
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
    // the counter must start at zero (a call that did not complete may have left it set)
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), s) != cudaSuccess) return MOE_ERR_CUDA;
    return moe::launch_route(x, T, D, Wr, bias, E, k, ids, gates, logits, ws, s);
}

