/*
 * moe.h — C ABI of the B200 routed-MoE expert pass.
 *
 * One MoE layer of a 512-expert, top-10 + 1-shared model, split in three
 * calls that the caller chains on one CUDA stream:
 *
 *   moe_route_topk      router logits, top-k expert ids and gates
 *   moe_expert_forward  expert-cache slot lookup (miss list out), then the
 *                       SwiGLU FFNs of every resident selected expert and of
 *                       the shared expert, over 2-/3-bit block-quantised
 *                       weights dequantised on the fly
 *   moe_combine         gate-weighted sum of the expert outputs + shared
 *                       expert (+ caller's partial for the misses) (+ residual)
 *
 * and, for decode batches (T <= 8), moe_layer_forward: the three in one launch
 * (without the misses' partial), with the same results.
 *
 * Sources: 512 routed experts per layer, 10 routed + 1 shared per token
 * (wiselychen RTX 5090 report, "30 秒定位"; greenbean-ai "Strata 如何讓 12GB
 * 顯卡跑 Qwen3.8-Flash-Next", §一).  The GPU runs the routing and the shared
 * expert, hot experts live in a VRAM cache and misses are computed elsewhere
 * (greenbean-ai §二; wiselychen report §2 "專家快取與 CPU／GPU 分工").  Weights
 * are 2-3.5 bit block-quantised (wiselychen report §1; greenbean-ai §四).
 * The SwiGLU form, the block layouts, the router normalisation and every
 * other detail the pages leave open are readings, stated at each declaration.
 *
 * Conventions for every call:
 *  - Pointers named x, Wr, ids, gates, logits, slot_table, expert_out,
 *    miss_list, miss_count, miss_partial, residual, out, ws and the pool's
 *    codes/scales are DEVICE pointers; the caller allocates and owns them.
 *    The library never allocates or frees, and synchronises only in
 *    moe_workspace_status.
 *  - bf16 and fp16 values are passed as uint16_t bit patterns.
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *    Argument and shape errors are returned synchronously and launch nothing;
 *    a failed launch returns MOE_ERR_CUDA.
 *  - Results are deterministic: no floating-point atomics, fixed summation
 *    orders; two identical calls give identical bits.
 *  - T == 0 is valid and launches nothing (miss_count is still zeroed).
 *  - Paths: the expert pass (moe_expert_forward) runs its decode path for
 *    T <= 24 (one token + MTP draft tokens; up to 8 tokens per launch, in
 *    token order) and its prefill path for T > 24.  The router
 *    (moe_route_topk) runs its decode path (CUDA cores) for T <= 24, in
 *    launches of n = min(T, 8) tokens, when (4 n + 8) D <= 196608 (every
 *    T <= 4; 8 tokens per launch up to D = 4864), and its prefill path
 *    (tensor cores) otherwise.  All paths compute the same function.
 *  - Kernels are launched with programmatic dependent launch: each may start
 *    while the previous kernel on the stream is finishing, and waits for it
 *    before reading the activations, ids, gates or expert_out it may have
 *    produced.  The layer's constants (Wr, bias, slot_table and the pool) may
 *    be read before that wait, to overlap their fetch with the previous kernel:
 *    they must not be written by the kernel launched immediately before the
 *    call (any earlier kernel, copy or event in between is fine).
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Identical to cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,   /* null pointer, bad size, misaligned pointer */
    MOE_ERR_UNSUPPORTED = -2,   /* shape outside the limits below */
    MOE_ERR_WORKSPACE = -3,     /* ws / expert_out smaller than the size query */
    MOE_ERR_CUDA = -4,          /* a CUDA call or launch failed */
    MOE_ERR_TIMEOUT = -5,       /* a bounded device-side wait gave up (moe_workspace_status) */
    MOE_ERR_RANGE = -6          /* a prefill activation outside the fp16 range (moe_workspace_status) */
} moe_status;

/*
 * Block formats (reading; the pages name Q2_0, IQ2_XS, IQ3_XXS ~3.06 bpw and
 * IQ3_S ~3.44 bpw without defining them).  Blocks run along the reduction
 * dimension K of every matrix.
 *   MOE_Q2_32  : 32 weights/block; 8 code bytes, weight j = bits [2j,2j+2) of
 *                the block's little-endian bit stream; fp16 s, fp16 m;
 *                w = fmaf(s, q, m).                        3.0 bits/weight
 *   MOE_Q3_32  : as Q2_32 with 12 code bytes, weight j = bits [3j,3j+3).
 *                                                          4.0 bits/weight
 *   MOE_Q3_S256: 256 weights/super-block; 96 code bytes, weight i = bits
 *                [3i,3i+3); 12 bytes of 6-bit sub-scales sc_j, j = 0..15, one
 *                per 16 weights, sub-block j = bits [6j,6j+6); fp16 d;
 *                w = d * (sc_j - 32) * (q - 4).            3.4375 bits/weight
 */
typedef enum moe_qformat { MOE_Q2_32 = 0, MOE_Q3_32 = 1, MOE_Q3_S256 = 2 } moe_qformat;

/*
 * A slot-mapped pool of quantised experts in device memory (the VRAM expert
 * cache of the wiselychen report §2).  Every slot holds one expert: gate Wg
 * [d_ff x d_model], up Wu [d_ff x d_model], down Wd [d_model x d_ff].
 *   codes  + s*slot_stride_codes : code planes gate | up | down, each row-major
 *                                  [rows][K/bw blocks][code bytes per block]
 *   scales + s*slot_stride_scales: Q2_32/Q3_32: (s, m) fp16 pairs (s first),
 *                                  planes gate | up | down, same block order;
 *                                  Q3_S256: 12-byte sub-scale planes gate | up |
 *                                  down, then fp16 d planes gate | up | down.
 * Strides are multiples of 256 bytes and at least moe_slot_code_bytes /
 * moe_slot_scale_bytes; codes and scales are 256-byte aligned.  shared_slot
 * is the always-resident shared expert of this layer.
 */
typedef struct moe_pool {
    int32_t fmt;          /* moe_qformat */
    int32_t d_model;      /* D */
    int32_t d_ff;         /* F */
    int32_t n_slots;
    int32_t shared_slot;
    int32_t reserved;     /* must be 0 */
    const void* codes;
    const void* scales;
    uint64_t slot_stride_codes;
    uint64_t slot_stride_scales;
} moe_pool;

/*
 * Shape limits (MOE_ERR_UNSUPPORTED otherwise):
 *   D % 256 == 0, 256 <= D <= 8192;  F % 128 == 0, 128 <= F <= 4096 (Q3_S256:
 *   F % 256 == 0);  1 <= k <= 16;  k <= E <= 1024;  0 <= T <= 65536.
 *   The expert pass's decode path (T <= 24) also keeps x (8 D bytes; 16 D for
 *   more than 4 tokens in a launch), two copies of h (16 F bytes; 32 F for T > 4) and at least two
 *   pipeline stages of 16 weight rows in 220 KB of shared memory per SM; the
 *   largest shapes do not fit and return MOE_ERR_UNSUPPORTED from
 *   moe_expert_forward (every shape with D + F <= 4096 fits).
 */

/* Bytes of one slot's codes / scale data (unpadded). */
size_t moe_slot_code_bytes(int fmt, int d_model, int d_ff);
size_t moe_slot_scale_bytes(int fmt, int d_model, int d_ff);

/* Workspace bytes for moe_route_topk / moe_expert_forward at these shapes. */
size_t moe_route_workspace_size(int T, int D, int E, int k);
size_t moe_workspace_size(int T, int D, int F, int E, int k, int fmt);
/* Bytes of the expert_out buffer moe_expert_forward fills and moe_combine reads. */
size_t moe_expert_out_size(int T, int D, int k);

/*
 * Router logits, top-k and gates (greenbean-ai §二: routing runs on the GPU;
 * wiselychen report "30 秒定位": top-10 of 512).
 *   x      bf16 [T][D] row-major, 16-byte aligned
 *   Wr     bf16 [E][D] row-major, 16-byte aligned
 *   bias   fp32 [E] or NULL (added to the logits before selection)
 *   ids    int32 [T][k] out: expert ids in rank order (larger logit first,
 *          equal logits: lower id first)
 *   gates  fp32 [T][k] out: exp(l_r - l_0) / sum_{r'<k} exp(l_r' - l_0)
 *          (reading: softmax restricted to the selected experts; sums to 1)
 *   logits fp32 [T][E] out, or NULL.  Decode path of the router: the
 *          canonical-order values below.  Prefill path: tensor-core values
 *          within the bound
 *          |l - canonical| <= 2^-12 * |x_t|_2 * |Wr_e|_2 (D <= 8192); the ids
 *          and gates always come from the canonical values.
 *   ws     device scratch of moe_route_workspace_size bytes, 256-byte
 *          aligned.  Its first 8 bytes must be zero before the first call
 *          with this buffer (e.g. zero it once at allocation); every completed
 *          call leaves them zero.  Calls sharing one ws must not overlap on
 *          the device.  Bytes 4..7 are the device error word: if a bounded
 *          device wait gave up (bit 0, MOE_ERR_TIMEOUT from
 *          moe_workspace_status), that call writes ids = -1 and gates = 0 for
 *          every token, and every later call on the same ws does the same
 *          until the caller zeroes the 8 bytes again.
 * The selection and the gates use logits in a canonical fp32 order: 32
 * partial sums, lane L accumulating fmaf over elements 256c + 8L + j (c
 * ascending, j = 0..7), then added pairwise (L with L+16, then +8, +4, +2,
 * +1), then + bias.  The ids are therefore reproducible bit for bit.
 */
moe_status moe_route_topk(const uint16_t* x, int T, int D, const uint16_t* Wr,
                          const float* bias, int E, int k, int32_t* ids, float* gates,
                          float* logits, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_route_topk without a workspace argument, for callers that cannot
 * allocate device memory themselves: code running under a host framework that
 * owns all device memory through a fixed, pre-sized arena and hands out no
 * scratch, or code that must not call cudaMalloc on its path.
 * The pages describe no such call; it is an addition of this library.
 *   Same arguments and results as moe_route_topk (decode path only).
 *   Scratch: a library-owned static device array of 16,640 bytes per GPU, held
 *   until the process exits; sizes beyond it (T > 4 or E > 1024) return
 *   MOE_ERR_UNSUPPORTED.  Nothing is allocated or freed.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.  Every call clears the array's block counter and device error
 *   word (8 bytes) with an async memset on `stream`; a call whose bounded
 *   device wait gave up writes ids = -1 and gates = 0.  All calls on a device
 *   share the array, which keeps the last call's logits: calls that overlap
 *   on the GPU (different streams) race and must be serialised by the caller.
 */
moe_status moe_route_topk_static(const uint16_t* x, int T, int D, const uint16_t* Wr,
                                 const float* bias, int E, int k, int32_t* ids, float* gates,
                                 float* logits, moe_stream_t stream);

/*
 * Slot lookup, miss list and expert FFNs.
 *   slot_table int32 [E]: expert id -> slot, -1 = not resident.  Any entry
 *          outside [0, n_slots) is treated as a miss.
 *   x      bf16 [T][D];  ids int32 [T][k] (from moe_route_topk or the caller;
 *          an id outside [0, E) is treated as a miss)
 *   expert_out   device buffer of moe_expert_out_size(T, D, k) bytes, 256-byte
 *          aligned: filled with one output row per (token, rank) hit and one
 *          per token for the shared expert, plus the row map moe_combine reads.
 *          Opaque to the caller.
 *   miss_list    int32 [T*k][3] out: (token, rank, expert) per miss, token-major
 *          then rank order (wiselychen report §2: misses go to the CPU, which
 *          computes them in place; here they are returned to the caller)
 *   miss_count   int32 [1] out
 *   ws     scratch of moe_workspace_size bytes, 256-byte aligned, distinct
 *          from the ws given to moe_route_topk.  Its first 1024 bytes must be
 *          zero before the first call with this buffer (zero it once at
 *          allocation); every completed call leaves them zero.  Calls sharing
 *          one ws must not overlap on the device.  Word 1 (bytes 4..7) is the
 *          device error word, read with moe_workspace_status:
 *            bit 0 (MOE_ERR_TIMEOUT): a bounded device wait gave up; the
 *              call's outputs are not valid, and every later call on this ws
 *              does no work until the caller zeroes its first 1024 bytes;
 *            bit 1 (MOE_ERR_RANGE): some x or h value has magnitude >= 65520,
 *              which the fp16 tensor-core operands cannot hold; the output
 *              rows of those tokens are not valid, the other rows are, and
 *              later calls are not affected (the bit stays set until the
 *              caller clears it).
 * Per expert (reading; the pages do not give the FFN form):
 *   h = bf16( silu(Wg x) * (Wu x) ),  y = Wd h,  fp32 accumulation.
 * Missed experts are not computed.
 * Operand precision (both paths): the tensor cores take fp16 operands with
 * fp32 accumulation.  Each weight is the exact weight of its block format
 * rounded once to fp16 (round to nearest even; see moe_debug_prefill_operand);
 * x and h (bf16 values) convert to fp16 exactly when their magnitude is below
 * 65520 (bit 1 of the error word otherwise).  Q3_S256 pools also need
 * |d*(sc-32)| < 65504.  Outputs are within the relative L2 bound of 1e-2 per
 * token of the exact-weight result.
 */
moe_status moe_expert_forward(const moe_pool* pool, const int32_t* slot_table, int E,
                              const uint16_t* x, int T, const int32_t* ids, int k,
                              void* expert_out, size_t expert_out_bytes,
                              int32_t* miss_list, int32_t* miss_count,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The expert pass with e4m3 tensor-core operands (a lossy variant of
 * moe_expert_forward's tensor-core path, T > 24; 1 <= T <= 24 returns
 * MOE_ERR_UNSUPPORTED and moe_workspace_size_fp8 returns 0 there, T = 0 only
 * clears miss_count).  Same arguments, results and error word; ws of
 * moe_workspace_size_fp8 bytes.
 * Operands: each weight is the exact weight of its block format times 64,
 * rounded once to fp16 and then to e4m3 (nearest even, saturating); x and h
 * are rounded to e4m3 (nearest even, saturating; magnitude >= 448 sets bit 1
 * of the error word); the products accumulate in fp32 and are scaled back by
 * 1/64.  The e4m3 roundings bound the accuracy, not the 1e-2 of
 * moe_expert_forward: on the 2,048-token synthetic workload the per-token
 * relative L2 error to the exact-weight result measured median 6.6e-2, max
 * 8.2e-2 (within 3e-3 of this variant's own definition).  Status as
 * moe_expert_forward.
 */
size_t moe_workspace_size_fp8(int T, int D, int F, int E, int k, int fmt);
moe_status moe_expert_forward_fp8(const moe_pool* pool, const int32_t* slot_table, int E,
                                  const uint16_t* x, int T, const int32_t* ids, int k,
                                  void* expert_out, size_t expert_out_bytes,
                                  int32_t* miss_list, int32_t* miss_count,
                                  void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Gate-weighted combine:
 *   out[t] = bf16( sum_{r<k, hit} gates[t][r] * y[t][r] + y_shared[t]
 *                  (+ miss_partial[t]) (+ residual[t]) )
 * summed in that order in fp32.  Gates are not renormalised over the hits
 * (reading: the caller adds the missed experts' contribution through
 * miss_partial, e.g. from a CPU pass over miss_list).
 *   expert_out   as filled by moe_expert_forward with the same T, D, k
 *   gates  fp32 [T][k];  miss_partial fp32 [T][D] or NULL;
 *   residual     bf16 [T][D] or NULL;  out bf16 [T][D] (may alias residual)
 */
moe_status moe_combine(const void* expert_out, const float* gates, int T, int D, int k,
                       const float* miss_partial, const uint16_t* residual,
                       uint16_t* out, moe_stream_t stream);

/*
 * One MoE layer for a small batch (T <= 8) in one launch: the results of
 *   moe_route_topk(x, ...) ; moe_expert_forward(...) ;
 *   moe_combine(expert_out, gates, T, D, k, NULL, residual, out)
 * bit for bit (ids, gates, expert_out rows of every hit and of the shared
 * expert, the row map, miss_list, miss_count and out).  The pages do not split
 * a decode layer into launches; this call is an addition of this library that
 * keeps the routing, the expert pass and the combine in one persistent kernel:
 * every CTA computes the logits of ceil(E / #SMs) experts, all CTAs meet at a
 * grid-wide barrier (a cooperative launch: one CTA per SM, all resident, so the
 * call waits for the whole GPU to be free of other work), every CTA then selects
 * every token's top-k itself; after the expert pass a second grid-wide
 * barrier, then each CTA combines a slice of the outputs.
 *   Arguments as in the three calls; residual bf16 [T][D] or NULL; out bf16
 *   [T][D] (may alias residual, not x).  Missed experts contribute nothing to
 *   out (to add them, call moe_combine again with miss_partial).
 *   ws     device scratch of moe_layer_workspace_size bytes, 256-byte aligned,
 *          zero before the first call (every completed call leaves its counters
 *          zero); word 1 is the device error word (moe_workspace_status).
 *          A call on a ws whose timeout bit is set does no work.  A bounded
 *          wait that gives up sets the timeout bit and the call writes ids -1
 *          and gates 0 (out is then not written).
 *   T > 8, or shapes whose routing does not fit the kernel's shared memory
 *   (the CTA's Wr rows and x as fp32 beside the expert pipeline; every shape
 *   with D + F <= 4096 and E <= 1024 fits): MOE_ERR_UNSUPPORTED, nothing
 *   launched (use the three calls).
 */
size_t moe_layer_workspace_size(int T, int D, int F, int E, int k, int fmt);
moe_status moe_layer_forward(const moe_pool* pool, const int32_t* slot_table, int E,
                             const uint16_t* x, int T, const uint16_t* Wr, const float* bias, int k,
                             int32_t* ids, float* gates, void* expert_out, size_t expert_out_bytes,
                             int32_t* miss_list, int32_t* miss_count,
                             const uint16_t* residual, uint16_t* out,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Test hook: dequantise one matrix of one slot to fp32, row-major
 * (matrix 0 = gate [F][D], 1 = up [F][D], 2 = down [D][F]).  Exact:
 * Q2_32/Q3_32 w = fmaf(s, q, m); Q3_S256 w = d*(sc-32)*(q-4).
 */
moe_status moe_dequantize(const moe_pool* pool, int slot, int matrix, float* out,
                          moe_stream_t stream);

/*
 * Device error word of a workspace (moe_route_topk's or moe_expert_forward's
 * ws): MOE_OK, MOE_ERR_TIMEOUT (bit 0) or MOE_ERR_RANGE (bit 1).  Unlike every
 * other call, this one synchronises `stream` (it waits for the work queued
 * on it) to read the word.
 */
moe_status moe_workspace_status(const void* ws, moe_stream_t stream);

/*
 * Test hook for the device error word: one device thread polls *flag (device
 * memory) until it equals `expect` or limit_us microseconds (1..1,000,000)
 * have passed; on the limit it sets bit 0 of ws's error word, as a bounded
 * wait of the expert pass does.  Returns at once on the device if that bit is
 * already set.
 */
moe_status moe_debug_wait_flag(const uint32_t* flag, uint32_t expect, uint32_t limit_us, void* ws,
                               moe_stream_t stream);

/*
 * Test hook: the weight operand of one tile of the prefill path's tensor-core
 * GEMM, exactly as the MMAs read it.  Runs the prefill GEMM kernel on a single
 * tile of `slot` (against zero rows) and copies its dequantised weight operand
 * back out of shared memory after each K = 64 round.
 *   gemm 1 (gate|up): weight rows 0..127 are gate features m0..m0+127 and rows
 *          128..255 the same up features (m0 % 128 == 0, m0 < d_ff), K = d_model;
 *   gemm 2 (down): weight rows are output features m0..m0+255 (m0 % 256 == 0,
 *          m0 < d_model), K = d_ff.
 *   dump   uint32 [K / 64][256][32] (device): word j of row r in round rr holds
 *          the fp16 pair (lo, hi) of weights K0 and K0 + 8, with c = j / 4,
 *          K0 = 64 rr + 16 (c / 2) + 4 (c % 2) + j % 4.
 *   ws     device scratch of moe_debug_operand_workspace_size bytes, 256-byte
 *          aligned (overwritten).
 * Each fp16 weight is the exact weight (moe_dequantize) rounded once to fp16.
 */
size_t moe_debug_operand_workspace_size(int d_model, int d_ff);
moe_status moe_debug_prefill_operand(const moe_pool* pool, int gemm, int slot, int m0, uint32_t* dump, void* ws,
                                     size_t ws_bytes, moe_stream_t stream);

/* Static text for a status code. */
const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
