/*
 * CPU oracle for the frozen AWQ routed-experts FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the smoke check and the bench's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * It is the plain definition of each step, written from the method's own
 * statements, accumulating in double:
 *
 *   ruda-tensor 0.21.34, src/packed_experts.rs
 *     - AwqExpertPayload: qweight I32 [E,K,N/8] (permuted words),
 *       qzeros I32 [E,K/group,N/8], scales FP32/FP16/BF16 [E,K/group,N],
 *       optional frozen bias [E,N]; AwqExpertOptions: N divisible by 8,
 *       complete input-channel groups, first global expert ID.
 *     - FrozenPackedExpertOps::packed_swiglu_forward: gate/up/down of the
 *       selected experts and a storage-rounded SwiGLU.
 *   ruda-tensor 0.21.33, src/frozen_awq.rs
 *     - FrozenAwqOps: the AWQ nibble order and the scale-dtype rounding of
 *       each coefficient are kept; output keeps the input's storage dtype;
 *       the input VJP applies the transpose of the same rounded coefficients.
 *   ruda-tensor 0.21.38, src/moe_exchange.rs
 *     - MoeDispatched / moe_dispatch: FP32 [tokens,top_k] weights, U32
 *       selected IDs, expert-sorted COPY rows with sorted U32 row_experts.
 *     - moe_combine: per token, ascending expert-ID combine.
 *     - moe_combine_backward: requested expert-row and FP32 weight VJPs.
 *     - moe_dispatch_backward: the COPY VJP sums the selected row seeds
 *       without applying routing weights again.
 *     - moe_dispatch_weights_backward: the logit VJP of the FP32 weights at a
 *       fixed selection.
 *
 * Readings taken where the pages are silent:
 *   - nibble order: slot s (bits 4s..4s+3 of the word read as unsigned)
 *     holds logical column 8w+P[s], P = {0,2,4,6,1,3,5,7};
 *   - coefficient W = RNE_sdt((q - z) * s): the product is exact, then
 *     rounded once to the scale dtype;
 *   - group of input row kk is kk / group; zeros unpack like weights;
 *   - selection: score = fp32(logit + selection bias); descending score,
 *     ties to the lower expert ID; weights are the softmax of the unbiased
 *     logits over the selected set (renormalize = 1), or the full softmax's
 *     probabilities of the selected experts (renormalize = 0);
 *   - rows inside one expert ascend by source token;
 *   - each stored tensor is rounded once (round to nearest even) to its
 *     storage dtype; h = RNE(silu(G) * U) from the rounded G and U.
 *
 * Storage dtype codes used by this file's callers: 0 = FP32, 1 = FP16,
 * 2 = BF16, 3 = FP64 (exact-math chaining of the tests; never rounded).
 * 16-bit tensors are passed as their bit patterns (uint16).
 *
 * ORACLE_MUTANT (a compile-time switch used only by tests/test_oracle_mutants.py;
 * 0 in every other build) plants one known mistake in one step, so that the
 * test can show that the pins below catch it.
 *
 * Parity pins: tests/test_oracle_pins.py (hand-worked words and
 * coefficients), tests/test_oracle_bruteforce.py (independent NumPy
 * dequantize-then-matmul), tests/test_oracle_invariants.py (routing and
 * dispatch invariants, adjoint identities, finite differences).
 */
#include <math.h>
#include <stdint.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#include <stdlib.h>
#include <string.h>

#define DT_F32 0
#define DT_F16 1
#define DT_BF16 2
#define DT_F64 3 /* exact-math chaining only: double storage, never rounded */

/* ------------------------------------------------------------------ */
/* Rounding a double to a binary floating format, nearest-even.        */
/* ------------------------------------------------------------------ */

/* Format parameters: p = significand bits including the implicit one,
 * emin = exponent of the smallest normal, emax = exponent of the largest
 * finite binade. */
static void fmt_params(int dt, int *p, int *emin, int *emax) {
    if (dt == DT_F16) { *p = 11; *emin = -14; *emax = 15; }
    else if (dt == DT_BF16) { *p = 8; *emin = -126; *emax = 127; }
    else { *p = 24; *emin = -126; *emax = 127; }
}

/* Nearest-even rounding of v onto the grid of format dt (gradual underflow,
 * overflow to infinity).  Returns the rounded value as a double (every value
 * of the three formats is exactly a double). */
double oracle_round(double v, int dt) {
    if (v == 0.0 || isnan(v) || isinf(v)) return v;
    int p, emin, emax;
    fmt_params(dt, &p, &emin, &emax);
    uint64_t bits;
    memcpy(&bits, &v, 8);
    int neg = (int)(bits >> 63);
    int bexp = (int)((bits >> 52) & 0x7FF);
    if (bexp == 0) return neg ? -0.0 : 0.0; /* double subnormal: far below every target */
    int e = bexp - 1023;                     /* v = 1.f * 2^e */
    uint64_t sig = (1ULL << 52) | (bits & ((1ULL << 52) - 1));
    int shift = 52 - (p - 1);                /* dropped low bits for a normal result */
    if (e < emin) shift += emin - e;         /* subnormal grid 2^(emin-p+1) */
    uint64_t q;
    if (shift > 53) {
        q = 0;                               /* below half the smallest step */
    } else {
        q = sig >> shift;
        uint64_t rem = sig & ((1ULL << shift) - 1);
        uint64_t half = 1ULL << (shift - 1);
        if (rem > half || (rem == half && (q & 1))) q += 1;
    }
    double out = ldexp((double)q, e - 52 + shift);
    double maxfin = ldexp(2.0 - ldexp(1.0, 1 - p), emax);
    if (out > maxfin) out = INFINITY;
    return neg ? -out : out;
}

/* Bits of an exactly representable value in format dt. */
uint32_t oracle_encode(double v, int dt) {
    double r = oracle_round(v, dt);
    if (dt == DT_F32 || dt == DT_BF16) {
        float f = (float)r; /* exact: r is on the FP32 (and so BF16) grid */
        uint32_t u;
        memcpy(&u, &f, 4);
        return dt == DT_F32 ? u : (u >> 16);
    }
    /* FP16 */
    uint32_t sign = signbit(r) ? 0x8000u : 0u;
    double a = fabs(r);
    if (isnan(r)) return 0x7E00u;
    if (isinf(a)) return sign | 0x7C00u;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {               /* subnormal: a = m * 2^-24 */
        return sign | (uint32_t)ldexp(a, 24);
    }
    int e;
    frexp(a, &e);                            /* a = f * 2^e, f in [0.5,1) */
    int ex = e - 1;                          /* a = 1.m * 2^ex */
    uint32_t mant = (uint32_t)(ldexp(a, -ex) * 1024.0 - 1024.0);
    return sign | ((uint32_t)(ex + 15) << 10) | mant;
}

double oracle_decode(uint32_t b, int dt) {
    if (dt == DT_F32) {
        float f;
        memcpy(&f, &b, 4);
        return (double)f;
    }
    if (dt == DT_BF16) {
        uint32_t u = b << 16;
        float f;
        memcpy(&f, &u, 4);
        return (double)f;
    }
    uint32_t sign = b & 0x8000u, ex = (b >> 10) & 0x1F, m = b & 0x3FF;
    double v;
    if (ex == 0) v = ldexp((double)m, -24);
    else if (ex == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 1024.0, (int)ex - 15);
    return sign ? -v : v;
}

static double load_val(const void *base, int dt, int64_t i) {
    if (dt == DT_F64) return ((const double *)base)[i];
    if (dt == DT_F32) return (double)((const float *)base)[i];
    return oracle_decode(((const uint16_t *)base)[i], dt);
}

static void store_val(void *base, int dt, int64_t i, double v) {
    if (dt == DT_F64) {
        ((double *)base)[i] = v;
    } else if (dt == DT_F32) {
        uint32_t u = oracle_encode(v, DT_F32);
        memcpy((char *)base + 4 * i, &u, 4);
    } else {
        ((uint16_t *)base)[i] = (uint16_t)oracle_encode(v, dt);
    }
}

/* ------------------------------------------------------------------ */
/* AWQ word unpack and coefficient.                                    */
/* ------------------------------------------------------------------ */

/* Logical column held by nibble slot s of a word (the packing order). */
static const int PACK_ORDER[8] = {0, 2, 4, 6, 1, 3, 5, 7};

/* codes[j] = code of logical column 8w+j.  The word is read as unsigned. */
void oracle_unpack_word(uint32_t word, int32_t codes[8]) {
    for (int s = 0; s < 8; ++s)
        codes[ORACLE_MUTANT == 1 ? s : PACK_ORDER[s]] = (int32_t)((word >> (4 * s)) & 0xFu);
}

uint32_t oracle_pack_word(const int32_t codes[8]) {
    uint32_t w = 0;
    for (int s = 0; s < 8; ++s) w |= ((uint32_t)codes[PACK_ORDER[s]] & 0xFu) << (4 * s);
    return w;
}

/* W = RNE_sdt((q - z) * s); returns its value, and its bits in *bits. */
double oracle_coefficient(int32_t q, int32_t z, uint32_t scale_bits, int sdt, uint32_t *bits) {
    double s = oracle_decode(scale_bits, sdt);
    double exact = (double)(q - z) * s;      /* |q-z| <= 15: exact in double */
    double w = oracle_round(exact, sdt);
    if (ORACLE_MUTANT == 2) w = oracle_round(oracle_round(q * s, sdt) - oracle_round(z * s, sdt), sdt);
    if (bits) *bits = oracle_encode(w, sdt);
    return w;
}

/* Dequantize one expert's projection: W[kk*N + n] for kk < K, n < N.
 * qw: [K, N/8] words, qz: [K/g, N/8] words, sc: [K/g, N] scales. */
void oracle_dequant(const int32_t *qw, const int32_t *qz, const void *sc, int sdt,
                    int64_t K, int64_t N, int64_t g, double *W, uint32_t *Wbits) {
    int64_t NW = N / 8;
#pragma omp parallel for schedule(static)
    for (int64_t kk = 0; kk < K; ++kk) {
        int64_t grp = kk / g;
        int64_t zgrp = (ORACLE_MUTANT == 3 && grp + 1 < K / g) ? grp + 1 : grp;
        for (int64_t w = 0; w < NW; ++w) {
            int32_t qc[8], zc[8];
            oracle_unpack_word((uint32_t)qw[kk * NW + w], qc);
            oracle_unpack_word((uint32_t)qz[zgrp * NW + w], zc);
            for (int j = 0; j < 8; ++j) {
                int64_t n = 8 * w + j;
                uint32_t sb = (sdt == DT_F32) ? 0u : ((const uint16_t *)sc)[grp * N + n];
                if (sdt == DT_F32) memcpy(&sb, (const char *)sc + 4 * (grp * N + n), 4);
                uint32_t b;
                double c = oracle_coefficient(qc[j], zc[j], sb, sdt, &b);
                if (W) W[kk * N + n] = c;
                if (Wbits) Wbits[kk * N + n] = b;
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Routing and COPY dispatch.                                          */
/* ------------------------------------------------------------------ */

/* selected[t*k + j]: global IDs (expert_start + local), descending score,
 * ties to the lower ID.  weights[t*k + j] FP32.  Returns 0, or -1 on bad
 * arguments. */
int oracle_route(const float *logits, const float *sel_bias, int64_t T, int64_t E,
                 int32_t k, int32_t renormalize, uint32_t expert_start,
                 uint32_t *selected, float *weights) {
    if (k < 1 || k > E) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        char *taken = (char *)calloc((size_t)E, 1);
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)k);
        for (int32_t j = 0; j < k; ++j) {
            int64_t best = -1;
            float bs = 0.f;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                float s = sel_bias ? (float)(l[e] + sel_bias[e]) : l[e];
                /* NaN (invalid input) ranks as -inf, so a round still takes a
                 * defined expert; -0 and +0 are equal scores (a tie) */
                if (isnan(s)) s = -INFINITY;
                /* strictly greater keeps the lower ID on ties */
                if (best < 0 || s > bs || (ORACLE_MUTANT == 4 && s == bs)) { best = e; bs = s; }
            }
            taken[best] = 1;
            sel[j] = best;
            selected[t * k + j] = expert_start + (uint32_t)best;
        }
        if (renormalize) {
            double m = -INFINITY, den = 0.0;
            double *lb = (double *)malloc(sizeof(double) * (size_t)k);
            for (int32_t j = 0; j < k; ++j)
                lb[j] = (double)l[sel[j]] + ((ORACLE_MUTANT == 5 && sel_bias) ? (double)sel_bias[sel[j]] : 0.0);
            for (int32_t j = 0; j < k; ++j) m = fmax(m, lb[j]);
            for (int32_t j = 0; j < k; ++j) den += exp(lb[j] - m);
            for (int32_t j = 0; j < k; ++j)
                weights[t * k + j] = (float)(exp(lb[j] - m) / den);
            free(lb);
        } else {
            double m = -INFINITY, den = 0.0;
            for (int64_t e = 0; e < E; ++e) m = fmax(m, (double)l[e]);
            for (int64_t e = 0; e < E; ++e) den += exp((double)l[e] - m);
            for (int32_t j = 0; j < k; ++j)
                weights[t * k + j] = (float)(exp((double)l[sel[j]] - m) / den);
        }
        free(taken);
        free(sel);
    }
    return 0;
}

/* Stable expert-sorted order of the T*k assignments: by (expert, token).
 * offsets[E+1] (exclusive prefix of counts), row_experts[A] (global IDs),
 * src_token[A], row_of[T*k].  Returns 0, or -1 if an ID is outside
 * [expert_start, expert_start + E). */
int oracle_dispatch(const uint32_t *selected, int64_t T, int32_t k, int64_t E,
                    uint32_t expert_start, int32_t *offsets, uint32_t *row_experts,
                    int32_t *src_token, int32_t *row_of) {
    int64_t A = T * k;
    int64_t *count = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int64_t a = 0; a < A; ++a) {
        int64_t e = (int64_t)selected[a] - (int64_t)expert_start;
        if (e < 0 || e >= E) { free(count); return -1; }
        count[e] += 1;
    }
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (int32_t)count[e];
    int64_t *next = (int64_t *)malloc(sizeof(int64_t) * (size_t)E);
    for (int64_t e = 0; e < E; ++e) next[e] = offsets[e];
    /* tokens in ascending order: each expert's rows ascend by token */
    for (int64_t tt = 0; tt < T; ++tt) {
        int64_t t = ORACLE_MUTANT == 6 ? T - 1 - tt : tt;
        for (int32_t j = 0; j < k; ++j) {
            int64_t e = (int64_t)selected[t * k + j] - (int64_t)expert_start;
            int64_t r = next[e]++;
            row_experts[r] = selected[t * k + j];
            src_token[r] = (int32_t)t;
            row_of[t * k + j] = (int32_t)r;
        }
    }
    free(count);
    free(next);
    return 0;
}

/* values[r,:] = x[src_token[r],:], bit copies of elem_bytes-wide elements. */
void oracle_copy_rows(const void *x, int64_t H, int64_t elem_bytes, const int32_t *src_token,
                      int64_t A, void *values) {
    for (int64_t r = 0; r < A; ++r)
        memcpy((char *)values + r * H * elem_bytes, (const char *)x + (int64_t)src_token[r] * H * elem_bytes,
               (size_t)(H * elem_bytes));
}

/* ------------------------------------------------------------------ */
/* Grouped projection of selected rows.                                */
/* ------------------------------------------------------------------ */

/* The rows of expert e, in ascending order; returns their count. */
static int64_t rows_of_expert(const int32_t *row_expert, int64_t R, int64_t e, int64_t *list) {
    int64_t n = 0;
    for (int64_t r = 0; r < R; ++r)
        if (row_expert[r] == e) list[n++] = r;
    return n;
}

/* Rows are taken ROW_BLOCK at a time so that each row of W, once loaded,
 * serves the whole block; every output still takes its terms in order. */
#define ROW_BLOCK 16

/* Rows r with row_expert[r] == e: out[r,n] = sum_kk x[r,kk] * W[kk,n] (+ bias[n]),
 * accumulated in double; mode 0 stores RNE in odt, 1 the double sum, 2 the
 * double sum of magnitudes (see oracle_project). */
static void expert_rows_times_W(const void *x, int xdt, int64_t R, int64_t K, int64_t N,
                                const int32_t *row_expert, int64_t e, const double *W,
                                const void *be, int bdt, int mode, void *out, int odt) {
    int64_t *list = (int64_t *)malloc(sizeof(int64_t) * (size_t)(R > 0 ? R : 1));
    const int64_t nr = rows_of_expert(row_expert, R, e, list);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b0 = 0; b0 < nr; b0 += ROW_BLOCK) {
        const int64_t nb = nr - b0 < ROW_BLOCK ? nr - b0 : ROW_BLOCK;
        double *acc = (double *)calloc((size_t)(nb * N), sizeof(double));
        for (int64_t kk = 0; kk < K; ++kk) {
            const double *Wr = W + kk * N;
            for (int64_t i = 0; i < nb; ++i) {
                const double xv = load_val(x, xdt, list[b0 + i] * K + kk);
                double *a = acc + i * N;
                /* each a[n] takes its terms in kk order; the n lanes are independent */
                if (mode == 2) {
#pragma omp simd
                    for (int64_t n = 0; n < N; ++n) a[n] += fabs(xv * Wr[n]);
                } else {
#pragma omp simd
                    for (int64_t n = 0; n < N; ++n) a[n] += xv * Wr[n];
                }
            }
        }
        for (int64_t i = 0; i < nb; ++i) {
            const int64_t r = list[b0 + i];
            for (int64_t n = 0; n < N; ++n) {
                double b = (be && ORACLE_MUTANT != 7) ? load_val(be, bdt, n) : 0.0;
                double v = acc[i * N + n] + (mode == 2 ? fabs(b) : b);
                if (mode >= 1) ((double *)out)[r * N + n] = v;
                else store_val(out, odt, r * N + n, v);
            }
        }
        free(acc);
    }
    free(list);
}

/* Rows r with row_expert[r] == e: out[r,kk] = sum_n grad[r,n] W[kk,n]
 * (+ sum_n grad2[r,n] W2[kk,n]), one double accumulator per output taking
 * its terms in n order (grad's, then grad2's); modes as above.  The loops
 * run over n outside and kk inside (on W transposed) so that the kk lanes,
 * which are independent, can be vectorised without reordering any sum. */
static void add_rows_times_WT(const void *grad, int gdt, const int64_t *rows, int64_t nb, int64_t N, int64_t K,
                              const double *WT, int mode, double *acc) {
    for (int64_t n = 0; n < N; ++n) {
        const double *Wc = WT + n * K;
        for (int64_t i = 0; i < nb; ++i) {
            const double gv = load_val(grad, gdt, rows[i] * N + n);
            double *a = acc + i * K;
            if (mode == 2) {
#pragma omp simd
                for (int64_t kk = 0; kk < K; ++kk) a[kk] += fabs(gv * Wc[kk]);
            } else {
#pragma omp simd
                for (int64_t kk = 0; kk < K; ++kk) a[kk] += gv * Wc[kk];
            }
        }
    }
}

static double *transposed(const double *W, int64_t K, int64_t N) {
    double *WT = (double *)malloc(sizeof(double) * (size_t)(K * N));
    for (int64_t kk = 0; kk < K; ++kk)
        for (int64_t n = 0; n < N; ++n) WT[n * K + kk] = W[kk * N + n];
    return WT;
}

static void expert_rows_times_WT(const void *grad, int gdt, int64_t R, int64_t N, int64_t K,
                                 const int32_t *row_expert, int64_t e, const double *W,
                                 const void *grad2, const double *W2, int mode, void *out, int odt) {
    int64_t *list = (int64_t *)malloc(sizeof(int64_t) * (size_t)(R > 0 ? R : 1));
    const int64_t nr = rows_of_expert(row_expert, R, e, list);
    double *WT = transposed(W, K, N);
    double *W2T = (W2 && ORACLE_MUTANT != 9) ? transposed(W2, K, N) : NULL;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b0 = 0; b0 < nr; b0 += ROW_BLOCK) {
        const int64_t nb = nr - b0 < ROW_BLOCK ? nr - b0 : ROW_BLOCK;
        double *acc = (double *)calloc((size_t)(nb * K), sizeof(double));
        add_rows_times_WT(grad, gdt, list + b0, nb, N, K, WT, mode, acc);
        if (W2T) add_rows_times_WT(grad2, gdt, list + b0, nb, N, K, W2T, mode, acc);
        for (int64_t i = 0; i < nb; ++i)
            for (int64_t kk = 0; kk < K; ++kk) {
                const int64_t r = list[b0 + i];
                if (mode >= 1) ((double *)out)[r * K + kk] = acc[i * K + kk];
                else store_val(out, odt, r * K + kk, acc[i * K + kk]);
            }
        free(acc);
    }
    free(WT);
    free(W2T);
    free(list);
}

/* Rows r < R of x ([R,K] in dtype xdt) go through the projection of their
 * expert row_expert[r] (local index < E):
 *   acc[r,n] = sum_kk x[r,kk] * W[e,kk,n]  (+ bias[e,n])
 * mode 0: out is stored in odt, rounded once (RNE) from the double sum.
 * mode 1: out is double [R,N], no output rounding (exact-math mode; the
 *         coefficients stay rounded because they are the operator).
 * mode 2: out is double [R,N] = sum_kk |x[r,kk] * W[e,kk,n]| (+ |bias|):
 *         the magnitude that bounds the rounding error of the same sum
 *         accumulated in a shorter format (used by the parity tolerance).
 * Returns 0, -1 on a bad expert index, -2 when K is not a whole number of
 * groups or N is not a multiple of 8 (AwqExpertOptions: complete
 * input-channel groups, output width divisible by eight). */
int oracle_project(const void *x, int xdt, int64_t R, int64_t K, int64_t N,
                   const int32_t *row_expert, int64_t E,
                   const int32_t *qw, const int32_t *qz, const void *sc, int sdt,
                   const void *bias, int bdt, int64_t g, int mode, void *out, int odt) {
    if (g < 1 || K % g != 0 || N % 8 != 0) return -2; /* complete groups, 8 columns per word */
    for (int64_t r = 0; r < R; ++r)
        if (row_expert[r] < 0 || row_expert[r] >= E) return -1;
    int64_t NW = N / 8, G = K / g;
    size_t sbytes = (sdt == DT_F32) ? 4 : 2, bbytes = (bdt == DT_F32) ? 4 : 2;
    double *W = (double *)malloc(sizeof(double) * (size_t)(K * N));
    for (int64_t e = 0; e < E; ++e) {
        int any = 0;
        for (int64_t r = 0; r < R && !any; ++r) any = (row_expert[r] == e);
        if (!any) continue;
        oracle_dequant(qw + e * K * NW, qz + e * G * NW, (const char *)sc + (size_t)(e * G * N) * sbytes, sdt,
                       K, N, g, W, NULL);
        const void *be = bias ? (const void *)((const char *)bias + (size_t)(e * N) * bbytes) : NULL;
        expert_rows_times_W(x, xdt, R, K, N, row_expert, e, W, be, bdt, mode, out, odt);
    }
    free(W);
    return 0;
}

/* ------------------------------------------------------------------ */
/* NF4 payload: ruda-tensor 0.21.34, src/packed_experts.rs,             */
/* PackedExpertPayload::Nf4 ("original RUDA high-nibble-first flat-block */
/* NF4"; packed scales and codebook frozen).  The pages print no layout; */
/* the reading: the 4-bit NormalFloat data type of Dettmers et al.,      */
/* "QLoRA: Efficient Finetuning of Quantized LLMs" (2023): 16 code       */
/* values (the codebook, an input), one absmax scale per block of B      */
/* consecutive elements of the flattened weight.                         */
/*   codes  uint8 [K*N/2]: the logical [K,N] matrix, flat index          */
/*          f = kk*N + n; byte f/2, high nibble (bits 4..7) for even f,  */
/*          low nibble for odd f;                                        */
/*   absmax f32 [K*N/B]; codebook f32 [16];                              */
/*   W[kk,n] = RNE_cdt(codebook[q] * absmax[f / B]): the F32 x F32       */
/*   product (exact in double) rounded once to the coefficient dtype.    */
/* ------------------------------------------------------------------ */

int32_t oracle_nf4_code(const uint8_t *codes, int64_t f) {
    uint8_t b = codes[f / 2];
    int high_first = ORACLE_MUTANT == 15 ? 0 : 1;
    return ((f % 2 == 0) == high_first) ? (int32_t)(b >> 4) : (int32_t)(b & 0xF);
}

void oracle_nf4_dequant(const uint8_t *codes, const float *absmax, const float *codebook, int64_t K,
                        int64_t N, int64_t B, int cdt, double *W, uint32_t *Wbits) {
#pragma omp parallel for schedule(static)
    for (int64_t kk = 0; kk < K; ++kk)
        for (int64_t n = 0; n < N; ++n) {
            int64_t f = kk * N + n;
            double exact = (double)codebook[oracle_nf4_code(codes, f)] * (double)absmax[f / B];
            double w = oracle_round(exact, cdt);
            if (W) W[f] = w;
            if (Wbits) Wbits[f] = oracle_encode(w, cdt);
        }
}

/* Grouped projection with NF4 payloads (rows, modes and return codes as
 * oracle_project; -2 when K*N is odd or not a whole number of blocks). */
int oracle_nf4_project(const void *x, int xdt, int64_t R, int64_t K, int64_t N,
                       const int32_t *row_expert, int64_t E, const uint8_t *codes, const float *absmax,
                       const float *codebook, int64_t B, int cdt, const void *bias, int bdt, int mode,
                       void *out, int odt) {
    if (B < 2 || (K * N) % B != 0 || (K * N) % 2 != 0) return -2;
    for (int64_t r = 0; r < R; ++r)
        if (row_expert[r] < 0 || row_expert[r] >= E) return -1;
    size_t bbytes = (bdt == DT_F32) ? 4 : 2;
    double *W = (double *)malloc(sizeof(double) * (size_t)(K * N));
    for (int64_t e = 0; e < E; ++e) {
        int any = 0;
        for (int64_t r = 0; r < R && !any; ++r) any = (row_expert[r] == e);
        if (!any) continue;
        oracle_nf4_dequant(codes + e * (K * N / 2), absmax + e * (K * N / B), codebook, K, N, B, cdt, W, NULL);
        const void *be = bias ? (const void *)((const char *)bias + (size_t)(e * N) * bbytes) : NULL;
        expert_rows_times_W(x, xdt, R, K, N, row_expert, e, W, be, bdt, mode, out, odt);
    }
    free(W);
    return 0;
}

/* Input VJP through the same NF4 coefficients (one payload). */
int oracle_nf4_input_backward(const void *grad, int gdt, int64_t R, int64_t N, int64_t K,
                              const int32_t *row_expert, int64_t E, const uint8_t *codes,
                              const float *absmax, const float *codebook, int64_t B, int cdt, int mode,
                              void *out, int odt) {
    if (B < 2 || (K * N) % B != 0 || (K * N) % 2 != 0) return -2;
    for (int64_t r = 0; r < R; ++r)
        if (row_expert[r] < 0 || row_expert[r] >= E) return -1;
    double *W = (double *)malloc(sizeof(double) * (size_t)(K * N));
    for (int64_t e = 0; e < E; ++e) {
        int any = 0;
        for (int64_t r = 0; r < R && !any; ++r) any = (row_expert[r] == e);
        if (!any) continue;
        oracle_nf4_dequant(codes + e * (K * N / 2), absmax + e * (K * N / B), codebook, K, N, B, cdt, W, NULL);
        expert_rows_times_WT(grad, gdt, R, N, K, row_expert, e, W, NULL, NULL, mode, out, odt);
    }
    free(W);
    return 0;
}

/* h = RNE(silu(G) * U), silu(v) = v / (1 + exp(-v)), from stored G and U
 * (dtype dt); h is stored in odt (DT_F64: the unrounded value). */
void oracle_swiglu(const void *G, const void *U, int dt, int64_t n, void *h, int odt) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double gv = load_val(G, dt, i), uv = load_val(U, dt, i);
        double silu = gv / (1.0 + exp(-gv));
        if (ORACLE_MUTANT == 8) silu = 1.0 / (1.0 + exp(-gv));
        store_val(h, odt, i, silu * uv);
    }
}

/* Positions of token t's k selections in ascending expert-ID order. */
static void ascending_slots(const uint32_t *sel, int32_t k, int32_t *order) {
    for (int32_t j = 0; j < k; ++j) order[j] = j;
    for (int32_t a = 1; a < k; ++a) { /* insertion sort on the IDs */
        int32_t v = order[a], b = a - 1;
        while (b >= 0 && sel[order[b]] > sel[v]) { order[b + 1] = order[b]; --b; }
        order[b + 1] = v;
    }
}

/* out[t,:] = RNE(sum over selections in ascending expert ID of w * y[row]),
 * stored in odt (DT_F64: the unrounded sum). */
void oracle_combine(const void *y, int dt, const float *weights, const uint32_t *selected,
                    const int32_t *row_of, int64_t T, int64_t H, int32_t k, void *out, int odt) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        int32_t order[64];
        ascending_slots(selected + t * k, k, order);
        for (int64_t c = 0; c < H; ++c) {
            double acc = 0.0;
            for (int32_t i = 0; i < k; ++i) {
                int32_t j = order[i];
                acc += (ORACLE_MUTANT == 10 ? 1.0 : (double)weights[t * k + j]) *
                       load_val(y, dt, (int64_t)row_of[t * k + j] * H + c);
            }
            store_val(out, odt, t * H + c, acc);
        }
    }
}

/* Combine VJP.  dy[row_of[t,j],:] = RNE(w[t,j] * dOut[t,:]) (stored in
 * dy_dt; DT_F64: unrounded); dweights[t,j] = FP32(sum_c dOut[t,c] *
 * y[row_of[t,j],c]).  Either output may be NULL (not requested). */
void oracle_combine_backward(const void *d_out, const void *y, int dt, const float *weights,
                             const int32_t *row_of, int64_t T, int64_t H, int32_t k,
                             void *dy, float *dweights, int dy_dt) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t j = 0; j < k; ++j) {
            int64_t r = row_of[t * k + j];
            double w = (double)weights[t * k + j], dot = 0.0;
            for (int64_t c = 0; c < H; ++c) {
                double g = load_val(d_out, dt, t * H + c);
                if (dy) store_val(dy, dy_dt, r * H + c, w * g);
                dot += g * (ORACLE_MUTANT == 13 ? g : load_val(y, dt, r * H + c));
            }
            if (dweights) dweights[t * k + j] = (float)dot;
        }
    }
}

/* Input VJP of one (or two summed) grouped projections:
 *   dinput[r,kk] = sum_n grad[r,n] W[e,kk,n]  (+ sum_n grad2[r,n] W2[e,kk,n])
 * rounded once to odt (mode 0) or left in double (mode 1); mode 2 gives the
 * double sum of the products' magnitudes (see oracle_project). */
int oracle_input_backward(const void *grad, int gdt, int64_t R, int64_t N, int64_t K,
                          const int32_t *row_expert, int64_t E,
                          const int32_t *qw, const int32_t *qz, const void *sc, int sdt, int64_t g,
                          const void *grad2, const int32_t *qw2, const int32_t *qz2, const void *sc2,
                          int mode, void *out, int odt) {
    if (g < 1 || K % g != 0 || N % 8 != 0) return -2; /* complete groups, 8 columns per word */
    for (int64_t r = 0; r < R; ++r)
        if (row_expert[r] < 0 || row_expert[r] >= E) return -1;
    int64_t NW = N / 8, G = K / g;
    size_t sbytes = (sdt == DT_F32) ? 4 : 2;
    double *W = (double *)malloc(sizeof(double) * (size_t)(K * N));
    double *W2 = grad2 ? (double *)malloc(sizeof(double) * (size_t)(K * N)) : NULL;
    for (int64_t e = 0; e < E; ++e) {
        int any = 0;
        for (int64_t r = 0; r < R && !any; ++r) any = (row_expert[r] == e);
        if (!any) continue;
        oracle_dequant(qw + e * K * NW, qz + e * G * NW, (const char *)sc + (size_t)(e * G * N) * sbytes, sdt,
                       K, N, g, W, NULL);
        if (W2)
            oracle_dequant(qw2 + e * K * NW, qz2 + e * G * NW, (const char *)sc2 + (size_t)(e * G * N) * sbytes,
                           sdt, K, N, g, W2, NULL);
        expert_rows_times_WT(grad, gdt, R, N, K, row_expert, e, W, grad2, W2, mode, out, odt);
    }
    free(W);
    free(W2);
    return 0;
}

/* SwiGLU VJP from the stored G, U:  s = 1/(1+exp(-G)),
 *   dG = RNE(dh * U * s * (1 + G * (1 - s))),  dU = RNE(dh * G * s),
 * stored in odt (DT_F64: unrounded). */
void oracle_swiglu_backward(const void *dh, const void *G, const void *U, int dt, int64_t n,
                            void *dG, void *dU, int odt) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double d = load_val(dh, dt, i), gv = load_val(G, dt, i), uv = load_val(U, dt, i);
        double s = 1.0 / (1.0 + exp(-gv));
        store_val(dG, odt, i, d * uv * s * (ORACLE_MUTANT == 11 ? 1.0 : (1.0 + gv * (1.0 - s))));
        store_val(dU, odt, i, d * gv * s);
    }
}

/* COPY VJP: dx[t,:] = RNE(sum over selections in ascending expert ID of
 * dvalues[row_of[t,j],:]); routing weights are not applied.  Stored in odt
 * (DT_F64: the unrounded sum). */
void oracle_dispatch_backward(const void *dvalues, int dt, const uint32_t *selected,
                              const int32_t *row_of, int64_t T, int64_t H, int32_t k, void *dx,
                              int odt) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        int32_t order[64];
        ascending_slots(selected + t * k, k, order);
        for (int64_t c = 0; c < H; ++c) {
            double acc = 0.0;
            for (int32_t i = 0; i < (ORACLE_MUTANT == 14 ? 1 : k); ++i)
                acc += load_val(dvalues, dt, (int64_t)row_of[t * k + order[i]] * H + c);
            store_val(dx, odt, t * H + c, acc);
        }
    }
}

/* Fixed-selection logit VJP of the FP32 weights (FP32 output [T,E]).
 * renormalize = 1: w_j = softmax over the selected logits, so
 *   dl[s_j] = w_j (dw_j - sum_i w_i dw_i), 0 for unselected experts.
 * renormalize = 0: w_j = p[s_j] with p the full softmax, so
 *   dl[e] = p_e ([e selected] dw_e - sum_j p[s_j] dw_j).
 * The weights are recomputed in double from the logits; the selection bias
 * only chose the set and receives no gradient. */
void oracle_router_backward(const float *logits, const uint32_t *selected, const float *d_weights,
                            int64_t T, int64_t E, int32_t k, int32_t renormalize,
                            uint32_t expert_start, float *d_logits) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        double *dl = (double *)calloc((size_t)E, sizeof(double));
        double m = -INFINITY, den = 0.0, dot = 0.0;
        if (renormalize) {
            for (int32_t j = 0; j < k; ++j) m = fmax(m, (double)l[selected[t * k + j] - expert_start]);
            for (int32_t j = 0; j < k; ++j) den += exp((double)l[selected[t * k + j] - expert_start] - m);
            for (int32_t j = 0; j < k; ++j) {
                double w = exp((double)l[selected[t * k + j] - expert_start] - m) / den;
                dot += w * (double)d_weights[t * k + j];
            }
            for (int32_t j = 0; j < k; ++j) {
                int64_t e = selected[t * k + j] - expert_start;
                double w = exp((double)l[e] - m) / den;
                dl[e] = w * ((double)d_weights[t * k + j] - (ORACLE_MUTANT == 12 ? 0.0 : dot));
            }
        } else {
            for (int64_t e = 0; e < E; ++e) m = fmax(m, (double)l[e]);
            for (int64_t e = 0; e < E; ++e) den += exp((double)l[e] - m);
            for (int32_t j = 0; j < k; ++j) {
                int64_t e = selected[t * k + j] - expert_start;
                dot += exp((double)l[e] - m) / den * (double)d_weights[t * k + j];
            }
            for (int64_t e = 0; e < E; ++e) dl[e] = -exp((double)l[e] - m) / den * dot;
            for (int32_t j = 0; j < k; ++j) {
                int64_t e = selected[t * k + j] - expert_start;
                dl[e] += exp((double)l[e] - m) / den * (double)d_weights[t * k + j];
            }
        }
        for (int64_t e = 0; e < E; ++e) d_logits[t * E + e] = (float)dl[e];
        free(dl);
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
