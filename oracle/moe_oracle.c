/*
 * moe_oracle.c — plain, slow CPU oracle of the routed-MoE expert pass.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.  Everything here is
 * written from the definitions (see moe_oracle.h for the sources); nothing is
 * blocked, fused or reordered beyond what a definition states.  Floating-point
 * work is done in double except where a definition fixes fp32 (router logits,
 * dequantised weights) or bf16 (h and the layer output).
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* number formats                                                      */
/* ------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* IEEE binary16 -> float, from the field definitions (exact). */
float orc_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return (float)(sign ? -v : v);
}

/* Round a double to the nearest bfloat16 (ties to even), returning its bits.
 * bfloat16 keeps 8 significant bits; its smallest normal is 2^-126 and its
 * subnormal spacing 2^-133. */
uint16_t orc_bf16_rne(double v)
{
    if (isnan(v)) return 0x7fc0;
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    int e;
    frexp(a, &e);                       /* a = f * 2^e, 0.5 <= f < 1 */
    int E = e - 1;                      /* a = 1.xxx * 2^E */
    double quantum = (E < -126) ? ldexp(1.0, -133) : ldexp(1.0, E - 7);
    double r = rint(a / quantum) * quantum;   /* rint: nearest, ties to even */
    if (r >= ldexp(1.0, 128)) r = INFINITY;
    float f = (float)r;                 /* exact: r is a bfloat16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t bits = (uint16_t)(u >> 16);
    return (uint16_t)(bits | (v < 0 ? 0x8000 : 0));
}

/* Round a double to the nearest IEEE binary16 value (ties to even) and return
 * that value.  11 significant bits; smallest normal 2^-14, subnormal spacing
 * 2^-24; magnitudes that round above 65504 become infinite. */
static double f16_round(double v)
{
    if (isnan(v) || v == 0.0) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);
    int E = e - 1;
    double quantum = (E < -14) ? ldexp(1.0, -24) : ldexp(1.0, E - 10);
    double r = rint(a / quantum) * quantum;
    if (r > 65504.0) r = INFINITY;
    return v < 0 ? -r : r;
}

/* E4M3 (8-bit float: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities, S.1111.111 is NaN, largest finite 448 = 1.75 * 2^8, subnormals
 * m * 2^-9).  Round to nearest, ties to even, saturating at +-448; NaN -> 0x7f. */
uint8_t orc_e4m3_rne(double v)
{
    if (isnan(v)) return 0x7f;
    const uint8_t sign = (v < 0 || (v == 0.0 && signbit(v))) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7e);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int E = e - 1;                                   /* a = 1.xxx * 2^E */
    double quantum = (E < -6) ? ldexp(1.0, -9) : ldexp(1.0, E - 3);
    double r = rint(a / quantum) * quantum;          /* nearest, ties to even */
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return sign;
    frexp(r, &e);
    E = e - 1;
    if (E < -6)                                      /* subnormal: m * 2^-9 */
        return (uint8_t)(sign | (int)(r / ldexp(1.0, -9)));
    int m = (int)(r / ldexp(1.0, E - 3)) - 8;        /* 1.mmm */
    return (uint8_t)(sign | ((E + 7) << 3) | m);
}

double orc_e4m3_to_f64(uint8_t b)
{
    const int e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return (b & 0x80) ? -v : v;
}

static double e4m3_value(double v) { return orc_e4m3_to_f64(orc_e4m3_rne(v)); }

/* the fp16 value nearest to v (ties to even), exposed for the oracle's pins */
double orc_f16_round(double v) { return f16_round(v); }

/* ------------------------------------------------------------------ */
/* block formats                                                        */
/*                                                                     */
/* Reading (the pages name Q2_0 / IQ2 / IQ3 formats of ~2-3.5 bits per  */
/* weight but define none of them): every matrix of a slot is stored    */
/* structure-of-arrays, rows = output features, blocks along the        */
/* reduction dimension K, row-major (row r, block b at index r*nb + b).  */
/*   Q2_32 : codes 8 B/block, weight j = bits [2j, 2j+2) of the block's  */
/*           little-endian bit stream; meta 4 B/block = fp16 s, fp16 m;  */
/*           w = fmaf(s, q, m).                                          */
/*   Q3_32 : codes 12 B/block, weight j = bits [3j, 3j+3); meta as Q2.   */
/*   Q3_S256: codes 96 B/super-block, weight i = bits [3i, 3i+3);        */
/*           12 B of 6-bit sub-scales, sub-block j (16 weights) = bits   */
/*           [6j, 6j+6); fp16 d; w = d * (sc - 32) * (q - 4).            */
/* Within a slot the code planes are gate (F x D), up (F x D), down      */
/* (D x F) in that order.  The meta region holds the three (s,m) planes   */
/* in the same order; for Q3_S256 it holds the three sub-scale planes     */
/* followed by the three d planes.                                        */
/* ------------------------------------------------------------------ */

static int block_weights(int fmt) { return fmt == ORC_Q3_S256 ? 256 : 32; }
static int block_code_bytes(int fmt) { return fmt == ORC_Q2_32 ? 8 : (fmt == ORC_Q3_32 ? 12 : 96); }
static int code_bits(int fmt) { return fmt == ORC_Q2_32 ? 2 : 3; }

static void matrix_shape(int matrix, int D, int F, int* rows, int* K)
{
    if (matrix == 2) { *rows = D; *K = F; }
    else { *rows = F; *K = D; }
}

size_t orc_slot_code_bytes(int fmt, int D, int F)
{
    size_t blocks = 3 * (size_t)D * F / block_weights(fmt);
    return blocks * block_code_bytes(fmt);
}

size_t orc_slot_scale_bytes(int fmt, int D, int F)
{
    size_t blocks = 3 * (size_t)D * F / block_weights(fmt);
    if (fmt == ORC_Q3_S256) return blocks * (12 + 2);
    return blocks * 4;
}

/* bit n of a little-endian byte stream */
static int stream_bit(const uint8_t* p, size_t n) { return (p[n / 8] >> (n % 8)) & 1; }

static int stream_field(const uint8_t* p, size_t first_bit, int nbits)
{
    int v = 0;
    for (int i = 0; i < nbits; ++i) v |= stream_bit(p, first_bit + i) << i;
    return v;
}

static uint16_t load_u16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* One dequantised row of `matrix` of `slot` into out[K]. */
static void dequant_row(const orc_pool* P, int slot, int matrix, int row, float* out)
{
    int rows, K;
    matrix_shape(matrix, P->d_model, P->d_ff, &rows, &K);
    const int bw = block_weights(P->fmt), cb = block_code_bytes(P->fmt);
    const int nb = K / bw;
    const uint8_t* codes = P->codes + (size_t)slot * P->stride_codes;
    const uint8_t* meta = P->scales + (size_t)slot * P->stride_scales;
    /* plane offsets: gate, up (F x D each), then down (D x F); all three
     * planes hold the same number of blocks, F*D/bw. */
    size_t plane_blocks = (size_t)P->d_ff * P->d_model / bw;
    const uint8_t* cplane = codes + (size_t)matrix * plane_blocks * cb;
    for (int b = 0; b < nb; ++b) {
        size_t blk = (size_t)row * nb + b;
        const uint8_t* bc = cplane + blk * cb;
        if (P->fmt == ORC_Q3_S256) {
            const uint8_t* sc = meta + ((size_t)matrix * plane_blocks + blk) * 12;
            const uint8_t* dp = meta + 3 * plane_blocks * 12 + ((size_t)matrix * plane_blocks + blk) * 2;
            float d = orc_f16_to_f32(load_u16(dp));
            for (int i = 0; i < 256; ++i) {
                int q = stream_field(bc, (size_t)3 * i, 3);
                int s6 = stream_field(sc, (size_t)6 * (i / 16), 6);
                out[b * 256 + i] = d * (float)((s6 - 32) * (q - 4));   /* exact */
            }
        } else {
            const uint8_t* sm = meta + ((size_t)matrix * plane_blocks + blk) * 4;
            float s = orc_f16_to_f32(load_u16(sm));
            float m = orc_f16_to_f32(load_u16(sm + 2));
            int nbits = code_bits(P->fmt);
            for (int j = 0; j < 32; ++j) {
                int q = stream_field(bc, (size_t)nbits * j, nbits);
                out[b * 32 + j] = fmaf(s, (float)q, m);
            }
        }
    }
}

static int pool_ok(const orc_pool* P)
{
    if (!P || !P->codes || !P->scales) return 0;
    if (P->fmt < ORC_Q2_32 || P->fmt > ORC_Q3_S256) return 0;
    if (P->d_model <= 0 || P->d_ff <= 0 || P->n_slots <= 0) return 0;
    int bw = block_weights(P->fmt);
    if (P->d_model % bw || P->d_ff % bw) return 0;
    return 1;
}

int orc_dequant(const orc_pool* P, int slot, int matrix, float* out)
{
    if (!pool_ok(P) || slot < 0 || slot >= P->n_slots || matrix < 0 || matrix > 2 || !out) return -1;
    int rows, K;
    matrix_shape(matrix, P->d_model, P->d_ff, &rows, &K);
    for (int r = 0; r < rows; ++r) dequant_row(P, slot, matrix, r, out + (size_t)r * K);
    return 0;
}

/* ------------------------------------------------------------------ */
/* 1. router logits                                                    */
/*                                                                     */
/* Reading (canonical order): for each (token, expert) 32 partial sums */
/* acc_L, L = 0..31, start at +0.0f; for c = 0..D/256-1 and j = 0..7,   */
/* acc_L = fmaf(x[256c+8L+j], Wr[e][256c+8L+j], acc_L).  They are then   */
/* added pairwise: level 1 p[L] = acc[L] + acc[L+16] (L < 16), level 2   */
/* p[L] = p[L] + p[L+8] (L < 8), then +4, +2, +1; logit = p[0] (+ b[e])  */
/* in fp32.  bf16 -> fp32 is exact.                                     */
/* ------------------------------------------------------------------ */
int orc_router_logits(const uint16_t* x, int T, int D, const uint16_t* Wr,
                      const float* bias, int E, float* logits)
{
    if (!x || !Wr || !logits || T < 0 || D <= 0 || D % 256 || E <= 0) return -1;
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            float acc[32];
            for (int L = 0; L < 32; ++L) acc[L] = 0.0f;
            for (int c = 0; c < D / 256; ++c)
                for (int j = 0; j < 8; ++j)
                    for (int L = 0; L < 32; ++L) {
                        int i = 256 * c + 8 * L + j;
                        acc[L] = fmaf(bf16_to_f32(x[(size_t)t * D + i]),
                                      bf16_to_f32(Wr[(size_t)e * D + i]), acc[L]);
                    }
            for (int half = 16; half >= 1; half /= 2)
                for (int L = 0; L < half; ++L) acc[L] = acc[L] + acc[L + half];
            float l = acc[0];
            if (bias) l = l + bias[e];
            logits[(size_t)t * E + e] = l;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* 2. top-k and gates                                                  */
/*                                                                     */
/* Order: larger logit first, equal logits -> lower expert id first.   */
/* Gates (reading of "gates summing to 1 over the selected experts"):   */
/* g_r = exp(l_r - l_0) / sum_{r'<k} exp(l_r' - l_0), in double, i.e.    */
/* softmax restricted to the k selected logits.                         */
/* ------------------------------------------------------------------ */
typedef struct { float l; int e; } cand;

static int cand_cmp(const void* a, const void* b)
{
    const cand* x = (const cand*)a;
    const cand* y = (const cand*)b;
    if (x->l > y->l) return -1;
    if (x->l < y->l) return 1;
    return (x->e < y->e) ? -1 : (x->e > y->e);
}

int orc_topk_gates(const float* logits, int T, int E, int k, int32_t* ids, double* gates)
{
    if (!logits || !ids || T < 0 || E <= 0 || k <= 0 || k > E) return -1;
    cand* c = (cand*)malloc(sizeof(cand) * (size_t)E);
    if (!c) return -1;
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) { c[e].l = logits[(size_t)t * E + e]; c[e].e = e; }
        qsort(c, (size_t)E, sizeof(cand), cand_cmp);
        double l0 = c[0].l, z = 0.0;
        for (int r = 0; r < k; ++r) z += exp((double)c[r].l - l0);
        for (int r = 0; r < k; ++r) {
            ids[(size_t)t * k + r] = c[r].e;
            if (gates) gates[(size_t)t * k + r] = exp((double)c[r].l - l0) / z;
        }
    }
    free(c);
    return 0;
}

/* ------------------------------------------------------------------ */
/* 3. slot lookup and miss list                                        */
/*                                                                     */
/* slot = slot_table[id]; an entry outside [0, n_slots) (normally -1)  */
/* is a miss.  One miss entry (t, r, expert) per missed (token, rank),  */
/* token-major then rank order.                                          */
/* ------------------------------------------------------------------ */
int orc_slot_lookup(const int32_t* ids, int T, int k, const int32_t* slot_table, int E,
                    int n_slots, int32_t* slots, int32_t* miss_list)
{
    if (!ids || !slot_table || T < 0 || k <= 0) return -1;
    int n = 0;
    for (int t = 0; t < T; ++t)
        for (int r = 0; r < k; ++r) {
            int e = ids[(size_t)t * k + r];
            int s = (e >= 0 && e < E) ? slot_table[e] : -1;
            if (s < 0 || s >= n_slots) s = -1;
            if (slots) slots[(size_t)t * k + r] = s;
            if (s < 0) {
                if (miss_list) {
                    miss_list[3 * n + 0] = t;
                    miss_list[3 * n + 1] = r;
                    miss_list[3 * n + 2] = e;
                }
                ++n;
            }
        }
    return n;
}

/* ------------------------------------------------------------------ */
/* 5. one SwiGLU expert                                                 */
/*   gate_pre[f] = sum_i Wg[f][i] x[i],  up_pre[f] = sum_i Wu[f][i] x[i] */
/*   h[f] = bf16( silu(gate_pre) * up_pre ),  silu(z) = z / (1 + e^-z)   */
/*   y[d] = sum_f Wd[d][f] h[f]                                          */
/* (the FFN form and the bf16 rounding of h are readings; the pages     */
/* only say the GPU computes the cached experts)                         */
/* ------------------------------------------------------------------ */
int orc_expert(const orc_pool* P, int slot, const uint16_t* x, uint16_t* h_out, double* y)
{
    if (!pool_ok(P) || slot < 0 || slot >= P->n_slots || !x || !y) return -1;
    const int D = P->d_model, F = P->d_ff;
    float* rowg = (float*)malloc(sizeof(float) * (size_t)(D > F ? D : F));
    float* rowu = (float*)malloc(sizeof(float) * (size_t)(D > F ? D : F));
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    if (!rowg || !rowu || !h) { free(rowg); free(rowu); free(h); return -1; }
    for (int f = 0; f < F; ++f) {
        dequant_row(P, slot, 0, f, rowg);
        dequant_row(P, slot, 1, f, rowu);
        double g = 0.0, u = 0.0;
        for (int i = 0; i < D; ++i) {
            double xi = bf16_to_f32(x[i]);
            g += (double)rowg[i] * xi;
            u += (double)rowu[i] * xi;
        }
        double silu = g / (1.0 + exp(-g));
        uint16_t hb = orc_bf16_rne(silu * u);
        if (h_out) h_out[f] = hb;
        h[f] = bf16_to_f32(hb);
    }
    for (int d = 0; d < D; ++d) {
        dequant_row(P, slot, 2, d, rowg);
        double acc = 0.0;
        for (int f = 0; f < F; ++f) acc += (double)rowg[f] * h[f];
        y[d] = acc;
    }
    free(rowg); free(rowu); free(h);
    return 0;
}

/* The e4m3-operand variant of the expert (the library's lossy option; the
 * pages fix no such variant, its definition is this library's):
 *   weight operand  W8 = e4m3( fp16( 64 w ) )  (w the exact block weight)
 *   x operand       x8 = e4m3( x )
 *   gate_pre = sum W8g x8 / 64,  up_pre = sum W8u x8 / 64   (double)
 *   h8 = e4m3( silu(gate_pre) * up_pre )
 *   y[d] = sum_f W8d[d][f] h8[f] / 64                       (double)  */
int orc_expert_fp8(const orc_pool* P, int slot, const uint16_t* x, double* y)
{
    if (!pool_ok(P) || slot < 0 || slot >= P->n_slots || !x || !y) return -1;
    const int D = P->d_model, F = P->d_ff;
    float* rowg = (float*)malloc(sizeof(float) * (size_t)(D > F ? D : F));
    float* rowu = (float*)malloc(sizeof(float) * (size_t)(D > F ? D : F));
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    double* x8 = (double*)malloc(sizeof(double) * (size_t)D);
    if (!rowg || !rowu || !h || !x8) { free(rowg); free(rowu); free(h); free(x8); return -1; }
    for (int i = 0; i < D; ++i) x8[i] = e4m3_value(bf16_to_f32(x[i]));
    for (int f = 0; f < F; ++f) {
        dequant_row(P, slot, 0, f, rowg);
        dequant_row(P, slot, 1, f, rowu);
        double g = 0.0, u = 0.0;
        for (int i = 0; i < D; ++i) {
            g += e4m3_value(f16_round(64.0 * rowg[i])) * x8[i];
            u += e4m3_value(f16_round(64.0 * rowu[i])) * x8[i];
        }
        g /= 64.0;
        u /= 64.0;
        h[f] = e4m3_value(g / (1.0 + exp(-g)) * u);
    }
    for (int d = 0; d < D; ++d) {
        dequant_row(P, slot, 2, d, rowg);
        double acc = 0.0;
        for (int f = 0; f < F; ++f) acc += e4m3_value(f16_round(64.0 * rowg[f])) * h[f];
        y[d] = acc / 64.0;
    }
    free(rowg); free(rowu); free(h); free(x8);
    return 0;
}

/* ------------------------------------------------------------------ */
/* 1-6: one layer                                                       */
/*   out[t] = bf16( sum_{r<k, hit} g[t,r] y[t,r] + y_shared[t]          */
/*                  (+ miss_partial[t]) (+ residual[t]) )                 */
/* summed in that order, in double.  Missed experts are not computed    */
/* and gates are not renormalised over the hits (reading: the GPU-only   */
/* path leaves misses to the caller, who may pass their partial sum).    */
/* The shared expert has weight 1 and always sits in pool->shared_slot.  */
/* ------------------------------------------------------------------ */
static int moe_layer_impl(const orc_pool* P, const int32_t* slot_table, int E, int k,
                          const uint16_t* x, int T, const uint16_t* Wr, const float* bias,
                          const float* miss_partial, const uint16_t* residual,
                          uint16_t* out, float* logits_out, int32_t* ids_out, double* gates_out,
                          int32_t* slots_out, int32_t* miss_list, int n_threads, int fp8)
{
    if (!pool_ok(P) || !slot_table || !x || !Wr || !out || T < 0 || k <= 0 || k > E) return -1;
    if (P->shared_slot < 0 || P->shared_slot >= P->n_slots) return -1;
    const int D = P->d_model;
    float* logits = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * E);
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1) * k);
    double* gates = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * k);
    int32_t* slots = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1) * k);
    if (!logits || !ids || !gates || !slots) { free(logits); free(ids); free(gates); free(slots); return -1; }

    int rc = orc_router_logits(x, T, D, Wr, bias, E, logits);
    if (rc == 0) rc = orc_topk_gates(logits, T, E, k, ids, gates);
    int n_miss = (rc == 0) ? orc_slot_lookup(ids, T, k, slot_table, E, P->n_slots, slots, miss_list) : -1;
    if (rc != 0 || n_miss < 0) { free(logits); free(ids); free(gates); free(slots); return -1; }

    /* Every (token, rank) hit and every token's shared expert is evaluated on
     * its own (independently, in parallel); the sum per token then runs in the
     * fixed order: ranks ascending, shared, miss_partial, residual. */
    int failed = 0;
    const int per_tok = k + 1;
    double* ys = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * per_tok * D);
    if (!ys) { free(logits); free(ids); free(gates); free(slots); return -1; }
#ifdef _OPENMP
    int nt = n_threads > 0 ? n_threads : 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(+ : failed)
#endif
    for (int pr = 0; pr < T * per_tok; ++pr) {
        int t = pr / per_tok, r = pr % per_tok;
        int s = (r < k) ? slots[(size_t)t * k + r] : P->shared_slot;
        if (s < 0) continue;
        const int rc_e = fp8 ? orc_expert_fp8(P, s, x + (size_t)t * D, ys + (size_t)pr * D)
                             : orc_expert(P, s, x + (size_t)t * D, NULL, ys + (size_t)pr * D);
        if (rc_e != 0) failed += 1;
    }
    for (int t = 0; t < T && !failed; ++t) {
        for (int d = 0; d < D; ++d) {
            double v = 0.0;
            for (int r = 0; r < k; ++r)
                if (slots[(size_t)t * k + r] >= 0)
                    v += gates[(size_t)t * k + r] * ys[((size_t)t * per_tok + r) * D + d];
            v += ys[((size_t)t * per_tok + k) * D + d];
            if (miss_partial) v += (double)miss_partial[(size_t)t * D + d];
            if (residual) v += (double)bf16_to_f32(residual[(size_t)t * D + d]);
            out[(size_t)t * D + d] = orc_bf16_rne(v);
        }
    }
    free(ys);
    (void)n_threads;
    if (logits_out) memcpy(logits_out, logits, sizeof(float) * (size_t)T * E);
    if (ids_out) memcpy(ids_out, ids, sizeof(int32_t) * (size_t)T * k);
    if (gates_out) memcpy(gates_out, gates, sizeof(double) * (size_t)T * k);
    if (slots_out) memcpy(slots_out, slots, sizeof(int32_t) * (size_t)T * k);
    free(logits); free(ids); free(gates); free(slots);
    return failed ? -1 : n_miss;
}

int orc_moe_layer(const orc_pool* P, const int32_t* slot_table, int E, int k,
                  const uint16_t* x, int T, const uint16_t* Wr, const float* bias,
                  const float* miss_partial, const uint16_t* residual,
                  uint16_t* out, float* logits_out, int32_t* ids_out, double* gates_out,
                  int32_t* slots_out, int32_t* miss_list, int n_threads)
{
    return moe_layer_impl(P, slot_table, E, k, x, T, Wr, bias, miss_partial, residual, out, logits_out, ids_out,
                          gates_out, slots_out, miss_list, n_threads, 0);
}

int orc_moe_layer_fp8(const orc_pool* P, const int32_t* slot_table, int E, int k,
                      const uint16_t* x, int T, const uint16_t* Wr, const float* bias,
                      const float* miss_partial, const uint16_t* residual,
                      uint16_t* out, float* logits_out, int32_t* ids_out, double* gates_out,
                      int32_t* slots_out, int32_t* miss_list, int n_threads)
{
    return moe_layer_impl(P, slot_table, E, k, x, T, Wr, bias, miss_partial, residual, out, logits_out, ids_out,
                          gates_out, slots_out, miss_list, n_threads, 1);
}
