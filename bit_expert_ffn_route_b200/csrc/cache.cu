// cache.cu — keeping the expert cache in step with use (include/moe_cache.h):
// the popularity count kernel, the host-side admission/eviction plan and the
// copy of an expert's weights into a pool slot.
//
// The pages: the most used experts stay in VRAM and the cache follows the
// actual use (wiselychen RTX 5090 report §2 "專家快取與 CPU／GPU 分工");
// the engine learns which experts are hot while it runs, and the copy engine
// streams expert data over PCIe while the GPU computes (greenbean-ai "Strata
// 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next", §二).  The plan's policy is a
// reading of those passages: the pages give no algorithm.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "moe.h"
#include "moe_cache.h"

namespace {

// counts[e] += occurrences of e among the n ids (ids outside [0, E) skipped).
__global__ void __launch_bounds__(256) expert_hist_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                          uint32_t* __restrict__ counts) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int e = __ldg(ids + i);
        if (e >= 0 && e < E) atomicAdd(counts + e, 1u);
    }
}

bool fmt_valid(int fmt) { return fmt == MOE_Q2_32 || fmt == MOE_Q3_32 || fmt == MOE_Q3_S256; }

}  // namespace

extern "C" moe_status moe_expert_hist(const int32_t* ids, int T, int k, int E, uint32_t* counts,
                                      moe_stream_t stream) {
    if (T < 0 || k <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!ids || !counts) return MOE_ERR_INVALID_ARG;
    const long long n = (long long)T * k;
    if (n > (1ll << 30)) return MOE_ERR_UNSUPPORTED;
    const int blocks = (int)std::min<long long>((n + 255) / 256, 1024);
    expert_hist_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(ids, (int)n, E, counts);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_cache_plan(const float* score, int E, const int32_t* slot_table, const int32_t* slots,
                              int n_slots, float hysteresis, int max_moves, moe_cache_move* moves,
                              int32_t* new_slot_table) {
    if (!score || !slot_table || !new_slot_table || E <= 0 || n_slots < 0 || max_moves < 0) return MOE_ERR_INVALID_ARG;
    if (n_slots > 0 && !slots) return MOE_ERR_INVALID_ARG;
    if (max_moves > 0 && !moves) return MOE_ERR_INVALID_ARG;
    if (!(hysteresis >= 1.0f) || !std::isfinite(hysteresis)) return MOE_ERR_INVALID_ARG;
    if (new_slot_table == slot_table) return MOE_ERR_INVALID_ARG;
    for (int e = 0; e < E; ++e)
        if (!std::isfinite(score[e]) || score[e] < 0.0f) return MOE_ERR_INVALID_ARG;
    // position of each slot in `slots` (slots are distinct), and its occupant
    std::vector<std::pair<int32_t, int>> pos;     // (slot id, index in slots)
    pos.reserve(n_slots);
    for (int i = 0; i < n_slots; ++i) pos.emplace_back(slots[i], i);
    std::sort(pos.begin(), pos.end());
    for (int i = 1; i < n_slots; ++i)
        if (pos[i].first == pos[i - 1].first) return MOE_ERR_INVALID_ARG;
    auto index_of = [&](int32_t slot) -> int {
        auto it = std::lower_bound(pos.begin(), pos.end(), std::make_pair(slot, -1));
        return (it != pos.end() && it->first == slot) ? it->second : -1;
    };
    std::vector<int> occupant(n_slots, -1);
    std::vector<int> residents, candidates;
    for (int e = 0; e < E; ++e) {
        new_slot_table[e] = slot_table[e];
        if (slot_table[e] < 0) {
            if (slot_table[e] != -1) return MOE_ERR_INVALID_ARG;
            if (score[e] > 0.0f) candidates.push_back(e);
            continue;
        }
        const int i = index_of(slot_table[e]);
        if (i < 0 || occupant[i] >= 0) return MOE_ERR_INVALID_ARG;
        occupant[i] = e;
        residents.push_back(e);
    }
    // candidates: score desc, id asc; residents, weakest first: score asc, id desc
    std::sort(candidates.begin(), candidates.end(),
              [&](int a, int b) { return score[a] != score[b] ? score[a] > score[b] : a < b; });
    std::sort(residents.begin(), residents.end(),
              [&](int a, int b) { return score[a] != score[b] ? score[a] < score[b] : a > b; });
    int n_moves = 0, next_free = 0, next_weak = 0;
    for (int c : candidates) {
        if (n_moves >= max_moves) break;
        while (next_free < n_slots && occupant[next_free] >= 0) ++next_free;
        if (next_free < n_slots) {                       // a free slot, in the order of `slots`
            occupant[next_free] = c;
            new_slot_table[c] = slots[next_free];
            moves[n_moves++] = moe_cache_move{slots[next_free], -1, c};
            continue;
        }
        if (next_weak >= (int)residents.size()) break;
        const int r = residents[next_weak];
        if (!(score[c] > hysteresis * score[r])) break;  // later candidates are no stronger
        ++next_weak;
        const int32_t s = slot_table[r];
        new_slot_table[r] = -1;
        new_slot_table[c] = s;
        moves[n_moves++] = moe_cache_move{s, r, c};
    }
    return n_moves;
}

extern "C" moe_status moe_slot_fill(const moe_pool* pool, int slot, const void* host_codes,
                                    const void* host_scales, moe_stream_t stream) {
    if (!pool || !pool->codes || !pool->scales || !host_codes || !host_scales) return MOE_ERR_INVALID_ARG;
    if (!fmt_valid(pool->fmt) || pool->d_model <= 0 || pool->d_ff <= 0) return MOE_ERR_INVALID_ARG;
    if (slot < 0 || slot >= pool->n_slots) return MOE_ERR_INVALID_ARG;
    const size_t cb = moe_slot_code_bytes(pool->fmt, pool->d_model, pool->d_ff);
    const size_t sb = moe_slot_scale_bytes(pool->fmt, pool->d_model, pool->d_ff);
    if (pool->slot_stride_codes < cb || pool->slot_stride_scales < sb) return MOE_ERR_INVALID_ARG;
    // the pool is read-only to the kernels; this call is the one writer of a slot
    uint8_t* dc = static_cast<uint8_t*>(const_cast<void*>(pool->codes)) + (size_t)slot * pool->slot_stride_codes;
    uint8_t* ds = static_cast<uint8_t*>(const_cast<void*>(pool->scales)) + (size_t)slot * pool->slot_stride_scales;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(dc, host_codes, cb, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(ds, host_scales, sb, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}
