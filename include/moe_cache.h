/*
 * moe_cache.h — C ABI for keeping the expert cache (the pool's slots) in step
 * with use: a popularity count fed by the router's ids, a host-side plan of
 * admissions and evictions, and the copy of an expert's weights into a slot.
 *
 * The pages: hot experts stay in VRAM while the rest live in host RAM; the
 * cache follows the actual use, so that the experts kept on the GPU match the
 * current work (wiselychen RTX 5090 report §2 "專家快取與 CPU／GPU 分工", 93.4%
 * hit rate in a logged run); the engine learns from use which experts are hot
 * (~72% hit rate against ~50% for a fixed cache) and the GPU's copy engine
 * pulls expert data over PCIe while the GPU computes (greenbean-ai "Strata
 * 如何讓 12GB 顯卡跑 Qwen3.8-Flash-Next", §二).  The policy below is a reading:
 * the pages give no algorithm.
 *
 * A caller's loop per layer (one possible arrangement):
 *   1. after moe_route_topk: moe_expert_hist(ids, ..., counts) on the stream;
 *   2. every N steps: copy counts to the host, fold them into a score (e.g.
 *      score = decay * score + counts), zero counts;
 *   3. moe_cache_plan(score, slot_table, slots, ...) -> moves;
 *   4. for each move: mark the evicted expert missing in the device slot table
 *      (stream order, so later kernels miss it), then on a copy stream that
 *      waits for the kernels issued so far, moe_slot_fill(pool, move.slot,
 *      weights of move.admit); after the copy (an event), write
 *      slot_table[move.admit] = move.slot.
 */
#ifndef MOE_CACHE_H
#define MOE_CACHE_H

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Popularity count: counts[e] += #{(t, r) : ids[t][r] == e} for every id in
 * [0, E); other ids are skipped.  Misses count too (popularity concerns
 * every routed expert, resident or not).
 *   ids     int32 [T][k], device;  counts uint32 [E], device (the caller
 *           zeroes it; the call only adds)
 * Integer atomic adds: the result does not depend on their order.
 * T == 0 launches nothing.
 */
moe_status moe_expert_hist(const int32_t* ids, int T, int k, int E, uint32_t* counts,
                           moe_stream_t stream);

/* One planned move of moe_cache_plan. */
typedef struct moe_cache_move {
    int32_t slot;    /* the slot to fill */
    int32_t evict;   /* the expert leaving it, or -1 if the slot was free */
    int32_t admit;   /* the expert entering it */
} moe_cache_move;

/*
 * Plan admissions and evictions for one layer's experts.  Host function: it
 * reads and writes host memory only, and never touches the device.
 *   score[E]       popularity per expert, finite and >= 0 (e.g. decayed
 *                  counts from moe_expert_hist)
 *   slot_table[E]  the current map expert -> slot, or -1 (not resident)
 *   slots[n_slots] the distinct slots this layer may use; every slot named in
 *                  slot_table must be one of them (the shared expert's slot is
 *                  not among them: the shared expert is not in the table)
 *   hysteresis     >= 1: an expert replaces a resident one only if its score
 *                  is greater than hysteresis x the resident's score
 *   max_moves      at most this many moves are planned (>= 0)
 *   moves          out, room for max_moves entries (may be NULL if 0)
 *   new_slot_table out [E]: slot_table with the moves applied (distinct from
 *                  slot_table)
 * Policy: the non-resident experts with score > 0 are taken by decreasing
 * score, ties by increasing id.  Each takes a free slot (in the order of
 * `slots`) while there is one; then it replaces the weakest resident left
 * (lowest score, ties: highest id) if it passes the hysteresis test, and the
 * plan stops at the first one that does not.  Residents that stay keep their
 * slots.
 * Returns the number of moves (>= 0), or MOE_ERR_INVALID_ARG for a null
 * pointer, E <= 0, a negative or non-finite score, hysteresis < 1 or not
 * finite, repeated slots, or a table entry that is not in `slots` or shared
 * by two experts.
 */
int moe_cache_plan(const float* score, int E, const int32_t* slot_table, const int32_t* slots, int n_slots,
                   float hysteresis, int max_moves, moe_cache_move* moves, int32_t* new_slot_table);

/*
 * Copy one expert's packed weights from host memory into slot `slot` of the
 * pool (written through the pool's codes/scales pointers).
 *   host_codes   moe_slot_code_bytes(pool->fmt, D, F) bytes in the slot layout
 *                of moe.h; host_scales likewise moe_slot_scale_bytes bytes
 * Two asynchronous host-to-device copies on `stream`; with pinned host memory
 * they run on a copy engine alongside kernels on other streams.  The caller
 * orders them: no kernel that reads the slot may run at the same time (see
 * the loop above).  Returns MOE_ERR_INVALID_ARG for a bad pool, slot or null
 * pointer, MOE_ERR_CUDA if a copy cannot be issued.
 */
moe_status moe_slot_fill(const moe_pool* pool, int slot, const void* host_codes, const void* host_scales,
                         moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_CACHE_H */
