// kernels.cuh — launchers shared between the kernel files and the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "moe.h"

namespace moe {

// Layout of the opaque expert_out buffer:
//   int32 rowmap[T][k+1]  row index of the output row of (token, rank), -1 = miss;
//                         rank k is the shared expert
//   (256-byte aligned) rows: decode path (T <= 8) fp32 [T*(k+1)][D], indexed t*(k+1)+r;
//                         prefill path bf16 [T*(k+1)][D], expert-ordered
inline size_t rowmap_bytes(int T, int k) { return ((size_t)T * (k + 1) * 4 + 255) / 256 * 256; }
inline size_t expert_out_bytes(int T, int D, int k) {
    const size_t row = (T <= kDecodeLayoutMaxT) ? 4 : 2;     // fp32 rows (decode path) or bf16 rows (prefill)
    return rowmap_bytes(T, k) + (size_t)T * (k + 1) * D * row;
}

struct PoolView {
    const uint8_t* codes;
    const uint8_t* scales;
    size_t stride_c, stride_s;
    int fmt, D, F, n_slots, shared_slot;
};

moe_status launch_route(const uint16_t* x, int T, int D, const uint16_t* Wr, const float* bias, int E,
                        int k, int32_t* ids, float* gates, float* logits, void* ws, cudaStream_t s);
size_t route_workspace_bytes(int T, int D, int E, int k);
moe_status launch_route_prefill(const uint16_t* x, int T, int D, const uint16_t* Wr, const float* bias, int E, int k,
                                int32_t* ids, float* gates, float* logits, float* wnorm, uint32_t* err,
                                cudaStream_t s);

moe_status launch_decode_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x,
                                 int T, const int32_t* ids, int k, void* expert_out, int32_t* miss_list,
                                 int32_t* miss_count, void* ws, cudaStream_t s);
size_t decode_workspace_bytes(int T, int D, int F, int k);
moe_status launch_layer_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x, int T,
                                const uint16_t* Wr, const float* bias, int k, int32_t* ids, float* gates,
                                void* expert_out, int32_t* miss_list, int32_t* miss_count, const uint16_t* residual,
                                uint16_t* out, void* ws, cudaStream_t s);
size_t layer_workspace_bytes(int T, int D, int F, int E, int k);

moe_status launch_prefill_forward(const PoolView& P, const int32_t* slot_table, int E, const uint16_t* x,
                                  int T, const int32_t* ids, int k, void* expert_out, int32_t* miss_list,
                                  int32_t* miss_count, void* ws, cudaStream_t s, bool fp8);
size_t prefill_workspace_bytes(int T, int D, int F, int E, int k);
size_t prefill_operand_dump_ws_bytes(int D, int F);
moe_status launch_prefill_operand_dump(const PoolView& P, int gemm, int slot, int m0, uint32_t* dump, void* ws,
                                       cudaStream_t s);

moe_status launch_combine(const void* expert_out, const float* gates, int T, int D, int k,
                          const float* miss_partial, const uint16_t* residual, uint16_t* out, cudaStream_t s);

moe_status launch_dequantize(const PoolView& P, int slot, int matrix, float* out, cudaStream_t s);
moe_status launch_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t limit_us, uint32_t* err, cudaStream_t s);

}  // namespace moe
