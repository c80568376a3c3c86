// api.cu — the extern "C" entry points declared in include/moe.h: argument
// validation, workspace sizing and dispatch between the decode (T <= 4) and
// prefill (T > 4) paths.  No allocation, no synchronisation.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.cuh"
#include "moe.h"
#include "sync.cuh"

using namespace moe;

namespace {

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int block_weights(int fmt) { return fmt == MOE_Q3_S256 ? 256 : 32; }

bool fmt_ok(int fmt) { return fmt == MOE_Q2_32 || fmt == MOE_Q3_32 || fmt == MOE_Q3_S256; }

moe_status check_shapes(int T, int D, int E, int k) {
    if (T < 0 || D <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (D % 256 || D > 8192 || k > kMaxTopK || E < k || E > 1024 || T > 65536) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_pool(const moe_pool* pool, PoolView& v) {
    if (!pool || !pool->codes || !pool->scales) return MOE_ERR_INVALID_ARG;
    if (!fmt_ok(pool->fmt) || pool->reserved != 0) return MOE_ERR_INVALID_ARG;
    const int D = pool->d_model, F = pool->d_ff;
    if (D <= 0 || F <= 0 || pool->n_slots <= 0) return MOE_ERR_INVALID_ARG;
    if (D % 256 || D > 8192 || F % 128 || F > 4096) return MOE_ERR_UNSUPPORTED;
    if (pool->fmt == MOE_Q3_S256 && F % 256) return MOE_ERR_UNSUPPORTED;
    if (pool->shared_slot < 0 || pool->shared_slot >= pool->n_slots) return MOE_ERR_INVALID_ARG;
    if (!aligned(pool->codes, 256) || !aligned(pool->scales, 256)) return MOE_ERR_INVALID_ARG;
    if (pool->slot_stride_codes % 256 || pool->slot_stride_scales % 256) return MOE_ERR_INVALID_ARG;
    if (pool->slot_stride_codes < moe_slot_code_bytes(pool->fmt, D, F) ||
        pool->slot_stride_scales < moe_slot_scale_bytes(pool->fmt, D, F))
        return MOE_ERR_INVALID_ARG;
    v.codes = static_cast<const uint8_t*>(pool->codes);
    v.scales = static_cast<const uint8_t*>(pool->scales);
    v.stride_c = pool->slot_stride_codes;
    v.stride_s = pool->slot_stride_scales;
    v.fmt = pool->fmt;
    v.D = D;
    v.F = F;
    v.n_slots = pool->n_slots;
    v.shared_slot = pool->shared_slot;
    return MOE_OK;
}

// A failed launch also leaves its (non-sticky) error as the runtime's last
// error; the status reports it, so clear it for the caller's next CUDA call.
moe_status reported(moe_status st) {
    if (st == MOE_ERR_CUDA) (void)cudaGetLastError();
    return st;
}

}  // namespace

extern "C" {

size_t moe_slot_code_bytes(int fmt, int d_model, int d_ff) {
    if (!fmt_ok(fmt) || d_model <= 0 || d_ff <= 0) return 0;
    const size_t blocks = 3 * (size_t)d_model * d_ff / block_weights(fmt);
    return blocks * (fmt == MOE_Q2_32 ? 8 : (fmt == MOE_Q3_32 ? 12 : 96));
}

size_t moe_slot_scale_bytes(int fmt, int d_model, int d_ff) {
    if (!fmt_ok(fmt) || d_model <= 0 || d_ff <= 0) return 0;
    const size_t blocks = 3 * (size_t)d_model * d_ff / block_weights(fmt);
    return blocks * (fmt == MOE_Q3_S256 ? 14 : 4);
}

size_t moe_route_workspace_size(int T, int D, int E, int k) {
    if (check_shapes(T, D, E, k) != MOE_OK) return 0;
    return route_workspace_bytes(T, D, E, k);
}

size_t moe_workspace_size(int T, int D, int F, int E, int k, int fmt) {
    if (check_shapes(T, D, E, k) != MOE_OK || F <= 0 || !fmt_ok(fmt)) return 0;
    if (T <= kDecodeLayoutMaxT) return decode_workspace_bytes(T < kDecodeMaxT ? T : kDecodeMaxT, D, F, k);
    return prefill_workspace_bytes(T, D, F, E, k);
}

size_t moe_expert_out_size(int T, int D, int k) {
    if (T < 0 || D <= 0 || k <= 0) return 0;
    return expert_out_bytes(T, D, k);
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_RANGE: return "activation outside the fp16 range";
    }
    return "unknown status";
}

moe_status moe_route_topk(const uint16_t* x, int T, int D, const uint16_t* Wr, const float* bias, int E, int k,
                          int32_t* ids, float* gates, float* logits, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
    moe_status st = check_shapes(T, D, E, k);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!x || !Wr || !ids || !gates || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(Wr, 16) || !aligned(ws, 256) || (logits && !aligned(logits, 16)))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < route_workspace_bytes(T, D, E, k)) return MOE_ERR_WORKSPACE;
    return reported(launch_route(x, T, D, Wr, bias, E, k, ids, gates, logits, ws, (cudaStream_t)stream));
}

moe_status moe_expert_forward(const moe_pool* pool, const int32_t* slot_table, int E, const uint16_t* x, int T,
                              const int32_t* ids, int k, void* expert_out, size_t expert_out_bytes_,
                              int32_t* miss_list, int32_t* miss_count, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
    PoolView v;
    moe_status st = check_pool(pool, v);
    if (st != MOE_OK) return st;
    st = check_shapes(T, v.D, E, k);
    if (st != MOE_OK) return st;
    if (!miss_count) return MOE_ERR_INVALID_ARG;
    if (T == 0) return cuda_status(cudaMemsetAsync(miss_count, 0, sizeof(int32_t), (cudaStream_t)stream));
    if (!slot_table || !x || !ids || !expert_out || !miss_list || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(expert_out, 256) || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    if (expert_out_bytes_ < expert_out_bytes(T, v.D, k)) return MOE_ERR_WORKSPACE;
    if (ws_bytes < moe_workspace_size(T, v.D, v.F, E, k, v.fmt)) return MOE_ERR_WORKSPACE;
    if (T <= kDecodeLayoutMaxT)
        return reported(launch_decode_forward(v, slot_table, E, x, T, ids, k, expert_out, miss_list, miss_count, ws,
                                              (cudaStream_t)stream));
    return reported(launch_prefill_forward(v, slot_table, E, x, T, ids, k, expert_out, miss_list, miss_count, ws,
                                           (cudaStream_t)stream, false));
}

size_t moe_workspace_size_fp8(int T, int D, int F, int E, int k, int fmt) {
    if (check_shapes(T, D, E, k) != MOE_OK || F <= 0 || !fmt_ok(fmt) || T <= kDecodeLayoutMaxT) return 0;
    return prefill_workspace_bytes(T, D, F, E, k);
}

moe_status moe_expert_forward_fp8(const moe_pool* pool, const int32_t* slot_table, int E, const uint16_t* x, int T,
                                  const int32_t* ids, int k, void* expert_out, size_t expert_out_bytes_,
                                  int32_t* miss_list, int32_t* miss_count, void* ws, size_t ws_bytes,
                                  moe_stream_t stream) {
    PoolView v;
    moe_status st = check_pool(pool, v);
    if (st != MOE_OK) return st;
    st = check_shapes(T, v.D, E, k);
    if (st != MOE_OK) return st;
    if (!miss_count) return MOE_ERR_INVALID_ARG;
    if (T == 0) return cuda_status(cudaMemsetAsync(miss_count, 0, sizeof(int32_t), (cudaStream_t)stream));
    if (T <= kDecodeLayoutMaxT) return MOE_ERR_UNSUPPORTED;    // moe_combine reads the small-batch layout there
    if (!slot_table || !x || !ids || !expert_out || !miss_list || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(expert_out, 256) || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    if (expert_out_bytes_ < expert_out_bytes(T, v.D, k)) return MOE_ERR_WORKSPACE;
    if (ws_bytes < moe_workspace_size_fp8(T, v.D, v.F, E, k, v.fmt)) return MOE_ERR_WORKSPACE;
    return reported(launch_prefill_forward(v, slot_table, E, x, T, ids, k, expert_out, miss_list, miss_count, ws,
                                           (cudaStream_t)stream, true));
}

size_t moe_layer_workspace_size(int T, int D, int F, int E, int k, int fmt) {
    if (check_shapes(T, D, E, k) != MOE_OK || F <= 0 || !fmt_ok(fmt) || T > kDecodeMaxT) return 0;
    return layer_workspace_bytes(T, D, F, E, k);
}

moe_status moe_layer_forward(const moe_pool* pool, const int32_t* slot_table, int E, const uint16_t* x, int T,
                             const uint16_t* Wr, const float* bias, int k, int32_t* ids, float* gates,
                             void* expert_out, size_t expert_out_bytes_, int32_t* miss_list, int32_t* miss_count,
                             const uint16_t* residual, uint16_t* out, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
    PoolView v;
    moe_status st = check_pool(pool, v);
    if (st != MOE_OK) return st;
    st = check_shapes(T, v.D, E, k);
    if (st != MOE_OK) return st;
    if (T > kDecodeMaxT) return MOE_ERR_UNSUPPORTED;
    if (!miss_count) return MOE_ERR_INVALID_ARG;
    if (T == 0) return cuda_status(cudaMemsetAsync(miss_count, 0, sizeof(int32_t), (cudaStream_t)stream));
    if (!slot_table || !x || !Wr || !ids || !gates || !expert_out || !miss_list || !out || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(Wr, 16) || !aligned(expert_out, 256) || !aligned(ws, 256) ||
        !aligned(out, 16) || (residual && !aligned(residual, 16)))
        return MOE_ERR_INVALID_ARG;
    if (out == x) return MOE_ERR_INVALID_ARG;
    if (expert_out_bytes_ < expert_out_bytes(T, v.D, k)) return MOE_ERR_WORKSPACE;
    if (ws_bytes < layer_workspace_bytes(T, v.D, v.F, E, k)) return MOE_ERR_WORKSPACE;
    return reported(launch_layer_forward(v, slot_table, E, x, T, Wr, bias, k, ids, gates, expert_out, miss_list,
                                         miss_count, residual, out, ws, (cudaStream_t)stream));
}

moe_status moe_combine(const void* expert_out, const float* gates, int T, int D, int k, const float* miss_partial,
                       const uint16_t* residual, uint16_t* out, moe_stream_t stream) {
    if (T < 0 || D <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (D % 256 || D > 8192 || k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!expert_out || !gates || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned(expert_out, 256) || !aligned(out, 16) || (residual && !aligned(residual, 16)) ||
        (miss_partial && !aligned(miss_partial, 16)))
        return MOE_ERR_INVALID_ARG;
    return reported(launch_combine(expert_out, gates, T, D, k, miss_partial, residual, out, (cudaStream_t)stream));
}

moe_status moe_dequantize(const moe_pool* pool, int slot, int matrix, float* out, moe_stream_t stream) {
    PoolView v;
    moe_status st = check_pool(pool, v);
    if (st != MOE_OK) return st;
    if (slot < 0 || slot >= v.n_slots || matrix < 0 || matrix > 2 || !out) return MOE_ERR_INVALID_ARG;
    return reported(launch_dequantize(v, slot, matrix, out, (cudaStream_t)stream));
}

moe_status moe_workspace_status(const void* ws, moe_stream_t stream) {
    if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    uint32_t word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&word, static_cast<const char*>(ws) + 4, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    if (word & kErrTimeout) return MOE_ERR_TIMEOUT;
    if (word & kErrRange) return MOE_ERR_RANGE;
    return MOE_OK;
}

moe_status moe_debug_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t limit_us, void* ws,
                               moe_stream_t stream) {
    if (!flag || !ws || !aligned(flag, 4) || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    if (limit_us == 0 || limit_us > 1000000u) return MOE_ERR_INVALID_ARG;
    return reported(launch_wait_flag(flag, expect, limit_us, reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 4),
                                     (cudaStream_t)stream));
}

size_t moe_debug_operand_workspace_size(int d_model, int d_ff) {
    if (d_model <= 0 || d_ff <= 0) return 0;
    return prefill_operand_dump_ws_bytes(d_model, d_ff);
}

moe_status moe_debug_prefill_operand(const moe_pool* pool, int gemm, int slot, int m0, uint32_t* dump, void* ws,
                                     size_t ws_bytes, moe_stream_t stream) {
    PoolView v;
    moe_status st = check_pool(pool, v);
    if (st != MOE_OK) return st;
    if (gemm != 1 && gemm != 2) return MOE_ERR_INVALID_ARG;
    if (slot < 0 || slot >= v.n_slots || !dump || !ws || !aligned(ws, 256) || !aligned(dump, 4)) return MOE_ERR_INVALID_ARG;
    if (m0 < 0 || (gemm == 1 ? (m0 % 128 || m0 >= v.F) : (m0 % 256 || m0 >= v.D))) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < prefill_operand_dump_ws_bytes(v.D, v.F)) return MOE_ERR_WORKSPACE;
    return reported(launch_prefill_operand_dump(v, gemm, slot, m0, dump, ws, (cudaStream_t)stream));
}

}  // extern "C"
