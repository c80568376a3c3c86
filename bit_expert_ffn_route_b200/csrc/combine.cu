// combine.cu — gate-weighted combine of the expert outputs.
//
//   out[t] = bf16( sum_{r<k, hit} g[t,r] * y[t,r] + y_shared[t] (+ miss_partial[t]) (+ residual[t]) )
//
// summed in exactly that order in fp32 (deterministic: no atomics).  The pages
// say each token uses 10 routed experts plus 1 shared expert (wiselychen RTX
// 5090 report, "30 秒定位"); the gate weighting and the unweighted shared expert
// are readings.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

namespace moe {
namespace {

// Decode path rows are fp32; each thread handles 4 consecutive features.
__global__ void __launch_bounds__(256) combine_f32_kernel(const int32_t* __restrict__ rowmap,
                                                          const float* __restrict__ rows,
                                                          const float* __restrict__ gates, int T, int D, int k,
                                                          const float* __restrict__ mp,
                                                          const uint16_t* residual, uint16_t* out) {
    pdl_wait();
    const int t = blockIdx.y;
    const int d = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (d >= D) return;
    // The decode path writes the row of (t, r) at index t*(k+1) + r (the row
    // map holds that index for a hit, -1 for a miss) and the shared row at
    // t*(k+1) + k: load those rows together with the map and the gates (one
    // round trip); a map entry pointing elsewhere is followed with a second load.
    int row[kMaxTopK];
    float g[kMaxTopK];
    float4 y[kMaxTopK];
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) {
        row[r] = (r < k) ? __ldg(rowmap + t * (k + 1) + r) : -1;
        g[r] = (r < k) ? __ldg(gates + t * k + r) : 0.f;
        y[r] = (r < k) ? __ldg(reinterpret_cast<const float4*>(rows + (size_t)(t * (k + 1) + r) * D + d))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int srow = __ldg(rowmap + t * (k + 1) + k);
    float4 ys = __ldg(reinterpret_cast<const float4*>(rows + (size_t)(t * (k + 1) + k) * D + d));
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r)
        if (row[r] >= 0 && row[r] != t * (k + 1) + r)
            y[r] = __ldg(reinterpret_cast<const float4*>(rows + (size_t)row[r] * D + d));
    if (srow != t * (k + 1) + k) ys = __ldg(reinterpret_cast<const float4*>(rows + (size_t)srow * D + d));
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) {
        if (row[r] >= 0) {
            a0 = __fmaf_rn(g[r], y[r].x, a0); a1 = __fmaf_rn(g[r], y[r].y, a1);
            a2 = __fmaf_rn(g[r], y[r].z, a2); a3 = __fmaf_rn(g[r], y[r].w, a3);
        }
    }
    a0 += ys.x; a1 += ys.y; a2 += ys.z; a3 += ys.w;
    if (mp) {
        const float4 m = __ldg(reinterpret_cast<const float4*>(mp + (size_t)t * D + d));
        a0 += m.x; a1 += m.y; a2 += m.z; a3 += m.w;
    }
    if (residual) {
        const uint2 rv = *reinterpret_cast<const uint2*>(residual + (size_t)t * D + d);
        a0 += bf16lo(rv.x); a1 += bf16hi(rv.x); a2 += bf16lo(rv.y); a3 += bf16hi(rv.y);
    }
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_rne(a0) | ((uint32_t)f32_to_bf16_rne(a1) << 16);
    o.y = (uint32_t)f32_to_bf16_rne(a2) | ((uint32_t)f32_to_bf16_rne(a3) << 16);
    *reinterpret_cast<uint2*>(out + (size_t)t * D + d) = o;
}

// Prefill path rows are bf16 (expert-ordered); each thread handles 8 features.
__global__ void __launch_bounds__(256) combine_bf16_kernel(const int32_t* __restrict__ rowmap,
                                                           const uint16_t* __restrict__ rows,
                                                           const float* __restrict__ gates, int T, int D, int k,
                                                           const float* __restrict__ mp,
                                                           const uint16_t* residual, uint16_t* out) {
    pdl_wait();
    const int t = blockIdx.y;
    const int d = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (d >= D) return;
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = 0.f;
    for (int r = 0; r < k; ++r) {
        const int row = __ldg(rowmap + (size_t)t * (k + 1) + r);
        if (row < 0) continue;
        const float g = __ldg(gates + (size_t)t * k + r);
        const uint4 y = __ldg(reinterpret_cast<const uint4*>(rows + (size_t)row * D + d));
        const uint32_t yy[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[2 * i] = __fmaf_rn(g, bf16lo(yy[i]), a[2 * i]);
            a[2 * i + 1] = __fmaf_rn(g, bf16hi(yy[i]), a[2 * i + 1]);
        }
    }
    {
        const int row = __ldg(rowmap + (size_t)t * (k + 1) + k);
        const uint4 y = __ldg(reinterpret_cast<const uint4*>(rows + (size_t)row * D + d));
        const uint32_t yy[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) { a[2 * i] += bf16lo(yy[i]); a[2 * i + 1] += bf16hi(yy[i]); }
    }
    if (mp) {
#pragma unroll
        for (int i = 0; i < 8; i += 4) {
            const float4 m = __ldg(reinterpret_cast<const float4*>(mp + (size_t)t * D + d + i));
            a[i] += m.x; a[i + 1] += m.y; a[i + 2] += m.z; a[i + 3] += m.w;
        }
    }
    if (residual) {
        const uint4 rv = *reinterpret_cast<const uint4*>(residual + (size_t)t * D + d);
        const uint32_t rr[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) { a[2 * i] += bf16lo(rr[i]); a[2 * i + 1] += bf16hi(rr[i]); }
    }
    uint4 o;
    uint32_t* oo = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        oo[i] = (uint32_t)f32_to_bf16_rne(a[2 * i]) | ((uint32_t)f32_to_bf16_rne(a[2 * i + 1]) << 16);
    *reinterpret_cast<uint4*>(out + (size_t)t * D + d) = o;
}

}  // namespace

moe_status launch_combine(const void* expert_out, const float* gates, int T, int D, int k,
                          const float* miss_partial, const uint16_t* residual, uint16_t* out, cudaStream_t s) {
    const int32_t* rowmap = reinterpret_cast<const int32_t*>(expert_out);
    const char* rows = reinterpret_cast<const char*>(expert_out) + rowmap_bytes(T, k);
    cudaError_t e;
    if (T <= kDecodeLayoutMaxT) {
        e = launch_pdl(combine_f32_kernel, dim3((D / 4 + 127) / 128, T), dim3(128), 0, s, rowmap,
                       reinterpret_cast<const float*>(rows), gates, T, D, k, miss_partial, residual, out);
    } else {
        e = launch_pdl(combine_bf16_kernel, dim3((D / 8 + 255) / 256, T), dim3(256), 0, s, rowmap,
                       reinterpret_cast<const uint16_t*>(rows), gates, T, D, k, miss_partial, residual, out);
    }
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
