/*
 * moe_oracle.h — plain, slow CPU oracle of the routed-MoE expert pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA library: it re-implements the
 * block formats and every step from their definitions.
 *
 * What it computes (one MoE layer, per token; sources named beside each step):
 *   1. router logits over E experts      (greenbean-ai "Strata 如何讓 12GB 顯卡跑
 *      Qwen3.8-Flash-Next", §二: the GPU does the routing; wiselychen RTX 5090
 *      report, "30 秒定位": 512 experts per layer, 10 routed + 1 shared)
 *   2. top-k (k = 10 on the pages) and gates normalised over the k selected
 *   3. expert-cache slot lookup with a miss list (wiselychen report §2
 *      "專家快取與 CPU／GPU 分工": hot experts cached in VRAM, misses elsewhere)
 *   4. on-the-fly dequantisation of 2-/3-bit block formats (wiselychen report
 *      §1 "低位元量化"; greenbean-ai §四: Q2_0 ... IQ3_S at ~2-3.5 bits/weight)
 *   5. SwiGLU expert FFN (a reading: the pages do not name the FFN form)
 *   6. gate-weighted combine + the always-on shared expert
 *
 * Readings of points the pages leave open are stated at each function; the
 * canonical summation order of the router logits is one of them: it is what
 * makes the selected expert ids reproducible bit for bit.
 *
 * Parity status: every function here is pinned by CPU tests against values
 * fixed by hand, closed forms, brute force and invariants.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* block formats (values are the oracle's own enumeration) */
#define ORC_Q2_32   0  /* 32 weights/block, 2-bit codes, fp16 scale s + fp16 min m */
#define ORC_Q3_32   1  /* 32 weights/block, 3-bit codes (96-bit LSB-first stream), fp16 s + m */
#define ORC_Q3_S256 2  /* 256 weights/super-block, 3-bit codes, 16 6-bit sub-scales, fp16 d */

typedef struct orc_pool {
    int fmt, d_model, d_ff, n_slots, shared_slot;
    const uint8_t* codes;          /* slot s codes at codes + s*stride_codes */
    const uint8_t* scales;         /* slot s scale data at scales + s*stride_scales */
    size_t stride_codes, stride_scales;
} orc_pool;

size_t orc_slot_code_bytes(int fmt, int D, int F);
size_t orc_slot_scale_bytes(int fmt, int D, int F);

/* 1. logits[t*E+e] in the canonical fp32 order; bias may be NULL. */
int orc_router_logits(const uint16_t* x, int T, int D, const uint16_t* Wr,
                      const float* bias, int E, float* logits);
/* 2. ids (rank order: logit desc, id asc) and gates (double). */
int orc_topk_gates(const float* logits, int T, int E, int k, int32_t* ids, double* gates);
/* 3. slots[t*k+r]; miss_list (t, r, expert) triples, token-major then rank; returns count. */
int orc_slot_lookup(const int32_t* ids, int T, int k, const int32_t* slot_table, int E,
                    int n_slots, int32_t* slots, int32_t* miss_list);
/* 4. dequantise one matrix of one slot: matrix 0 = gate [F x D], 1 = up [F x D],
 *    2 = down [D x F]; out is row-major fp32. */
int orc_dequant(const orc_pool* pool, int slot, int matrix, float* out);
/* 5. one expert on one token: h (bf16 bits, may be NULL) and y (double [D]). */
int orc_expert(const orc_pool* pool, int slot, const uint16_t* x, uint16_t* h, double* y);
/* 1-6 for T tokens.  miss_partial (fp32 [T*D]) and residual (bf16 [T*D]) may be NULL.
 * Outputs: out bf16 [T*D]; logits [T*E], ids/gates/slots [T*k], miss_list [T*k*3]
 * (each may be NULL except out); returns the miss count, or < 0 on bad arguments. */
int orc_moe_layer(const orc_pool* pool, const int32_t* slot_table, int E, int k,
                  const uint16_t* x, int T, const uint16_t* Wr, const float* bias,
                  const float* miss_partial, const uint16_t* residual,
                  uint16_t* out, float* logits, int32_t* ids, double* gates,
                  int32_t* slots, int32_t* miss_list, int n_threads);

/* The e4m3-operand variant (weights e4m3(fp16(64 w)), x and h e4m3, products
 * in double scaled by 1/64): one expert, and 1-6 for T tokens with the same
 * arguments and results as orc_moe_layer. */
int orc_expert_fp8(const orc_pool* pool, int slot, const uint16_t* x, double* y);
int orc_moe_layer_fp8(const orc_pool* pool, const int32_t* slot_table, int E, int k,
                      const uint16_t* x, int T, const uint16_t* Wr, const float* bias,
                      const float* miss_partial, const uint16_t* residual,
                      uint16_t* out, float* logits, int32_t* ids, double* gates,
                      int32_t* slots, int32_t* miss_list, int n_threads);

/* helpers exposed for the oracle's own pins */
uint16_t orc_bf16_rne(double v);
float    orc_f16_to_f32(uint16_t h);
uint8_t  orc_e4m3_rne(double v);         /* nearest even, saturating at +-448 */
double   orc_e4m3_to_f64(uint8_t b);
double   orc_f16_round(double v);         /* nearest fp16 value, ties to even */

#ifdef __cplusplus
}
#endif
#endif
