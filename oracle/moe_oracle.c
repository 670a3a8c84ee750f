/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle for the forward pass of a
 * Mixture-of-Experts SwiGLU FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA product path
 * shares no code with it and never calls it.
 *
 * What it computes, per token t (each step is the plain definition, no
 * blocking, fusion or reordering beyond what the definition states):
 *
 *   1. router logits  l_e = sum_i x_ti * Wr[e][i]  (+ b_e)
 *        "Fused MoE Triton kernel: 5 launches instead of 24" page, list of
 *        fused steps, first item (top-k routing weights); "CUDA: fuse shared
 *        experts into MMVQ" page, section on shared experts (the router picks
 *        the top-k experts per token).
 *   2. p = softmax(l) over all E experts.
 *   3. the k experts with the largest logits, ties to the lower index.
 *   4. w_j = p_j / sum over the selected experts of p  (renormalisation).
 *   5. dispatch: tokens grouped per expert (counts, exclusive offsets and a
 *        stable slot order, ascending token index inside each expert) --
 *        Triton-kernel page, second fused step and the launch table's
 *        dispatch row.
 *   6. each selected expert and every shared expert computes
 *        FFN(x) = Wd (SiLU(Wg x) * (Wu x)),  SiLU(z) = z / (1 + e^-z)
 *        -- Triton-kernel page, third fused step; MMVQ page, shared experts
 *        are always active and add a fixed amount of work per token.
 *   7. out_t = sum_j w_j FFN_j(x_t) + sum_s FFN_s(x_t)  (shared weight 1)
 *        -- Triton-kernel page, fourth fused step (weighted aggregation).
 *
 * The weights are read in the exact formats the GPU sees: bf16 values,
 * fp32 router, and Q4_0 blocks dequantised here as w = d * (q - 8) from the
 * canonical 18-byte blocks (fp16 scale d, then 16 bytes; byte j holds
 * element j in its low nibble and element j+16 in its high nibble), and Q8_0
 * blocks as w = d * q from the canonical 34-byte blocks (fp16 scale d, then
 * 32 signed bytes q, element j in byte j; the 5090 page names q8_0 among the
 * formats of the model it measures), and Q5_0 blocks as w = d * (q - 16) from
 * the canonical 22-byte blocks (fp16 scale d, a little-endian 32-bit word qh
 * of fifth bits, then 16 bytes of low nibbles as in Q4_0; element j takes
 * bit j of qh as its fifth bit; q5_0 is in the same list of formats), and
 * q6_K super-blocks as w = d * sc * (q - 32) from the canonical 210-byte
 * super-blocks of 256 weights (see q6_k_row; q6_K is in the same list).
 * Every dequantised value is exact in double precision.
 *
 * Layouts (row-major, reduction dimension contiguous):
 *   x [T][d] bf16 bits; Wr [E][d] fp32; b [E] fp32 or NULL
 *   routed gate/up [E][F][d], down [E][d][F]; shared [S][Fs][d], [S][d][Fs]
 *   Q4_0: a row of K weights is K/32 blocks of 18 bytes.
 *   Q8_0: a row of K weights is K/32 blocks of 34 bytes.
 *   Q5_0: a row of K weights is K/32 blocks of 22 bytes.
 *   q6_K: a row of K weights is K/256 super-blocks of 210 bytes.
 *   BF16_F16DOWN: gate/up as bf16 bits, every down matrix (routed and shared)
 *   as IEEE fp16 bits [.][d][F] -- the bf16 weights rounded to fp16 once, so
 *   that the prefill down GEMM can take h in fp16 (see the kernels).
 *
 * The pages print no worked example for the layer output, so the tests pin
 * every function here against what the mathematics fixes instead: brute-force
 * evaluation on tiny inputs, closed forms (k = E dense mixture, one-hot
 * router, a single dense SwiGLU FFN), library routines (numpy matmul, IEEE
 * half/bfloat16 decoding) and hand-derived values under tests/golden/.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_WFMT_BF16 0
#define ORACLE_WFMT_Q4_0 1
#define ORACLE_WFMT_Q8_0 2
#define ORACLE_WFMT_Q5_0 3
#define ORACLE_WFMT_Q6_K 4
#define ORACLE_WFMT_BF16_F16DOWN 5   /* gate/up bf16, down (routed and shared) fp16 */
#define ORACLE_ROWS_F16 100          /* internal: rows of fp16 bit patterns */

/* bfloat16 is the top half of an IEEE binary32. */
double oracle_bf16_to_f64(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_fp16_to_f64(uint16_t h) {
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1024.0 + (double)m, e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return s ? -v : v;
}

/* Dequantise one row of K weights stored as canonical Q4_0 blocks. */
static void q4_0_row(const uint8_t* blocks, int64_t K, double* out) {
    for (int64_t b = 0; b < K / 32; ++b) {
        const uint8_t* blk = blocks + b * 18;
        uint16_t hd = (uint16_t)(blk[0] | (blk[1] << 8));
        double dsc = oracle_fp16_to_f64(hd);
        for (int j = 0; j < 16; ++j) {
            int lo = blk[2 + j] & 0x0f;
            int hi = blk[2 + j] >> 4;
            out[b * 32 + j] = dsc * (double)(lo - 8);
            out[b * 32 + j + 16] = dsc * (double)(hi - 8);
        }
    }
}

/* Dequantise one row of K weights stored as canonical Q8_0 blocks. */
static void q8_0_row(const uint8_t* blocks, int64_t K, double* out) {
    for (int64_t b = 0; b < K / 32; ++b) {
        const uint8_t* blk = blocks + b * 34;
        uint16_t hd = (uint16_t)(blk[0] | (blk[1] << 8));
        double dsc = oracle_fp16_to_f64(hd);
        for (int j = 0; j < 32; ++j) {
            int q = blk[2 + j] < 128 ? (int)blk[2 + j] : (int)blk[2 + j] - 256;  /* two's complement */
            out[b * 32 + j] = dsc * (double)q;
        }
    }
}

/* Dequantise one row of K weights stored as canonical Q5_0 blocks. */
static void q5_0_row(const uint8_t* blocks, int64_t K, double* out) {
    for (int64_t b = 0; b < K / 32; ++b) {
        const uint8_t* blk = blocks + b * 22;
        uint16_t hd = (uint16_t)(blk[0] | (blk[1] << 8));
        double dsc = oracle_fp16_to_f64(hd);
        uint32_t qh = (uint32_t)blk[2] | ((uint32_t)blk[3] << 8) | ((uint32_t)blk[4] << 16) |
                      ((uint32_t)blk[5] << 24);
        for (int j = 0; j < 16; ++j) {
            int lo = (blk[6 + j] & 0x0f) | (int)(((qh >> j) & 1u) << 4);
            int hi = (blk[6 + j] >> 4) | (int)(((qh >> (j + 16)) & 1u) << 4);
            out[b * 32 + j] = dsc * (double)(lo - 16);
            out[b * 32 + j + 16] = dsc * (double)(hi - 16);
        }
    }
}

/* Dequantise one row of K weights stored as canonical q6_K super-blocks (K a
 * multiple of 256; 210 bytes per 256 weights: ql[128] low 4 bits, qh[64]
 * high 2 bits, 16 signed 8-bit sub-block scales, then a little-endian fp16
 * super-block scale d; the 5090 page names q6_K among the formats of the
 * model it measures and prints no layout -- this is the reading taken).
 * Element i of a super-block: h = i / 128 (which half), r = i % 128,
 * c = r / 32 (which quarter of the half), l = r % 32.  Its low 4 bits are
 * the low nibble (c = 0, 1) or the high nibble (c = 2, 3) of byte
 * ql[64 h + l] (c even) or ql[64 h + 32 + l] (c odd); its high 2 bits are
 * bits 2c, 2c+1 of qh[32 h + l]; its sub-block is i / 16.
 * weight = d * sc[i / 16] * (q - 32), q = low + 16 * high in 0..63. */
static void q6_k_row(const uint8_t* blocks, int64_t K, double* out) {
    for (int64_t b = 0; b < K / 256; ++b) {
        const uint8_t* blk = blocks + b * 210;
        const uint8_t* ql = blk;
        const uint8_t* qh = blk + 128;
        const uint8_t* sc = blk + 192;
        uint16_t hd = (uint16_t)(blk[208] | (blk[209] << 8));
        double dsc = oracle_fp16_to_f64(hd);
        for (int i = 0; i < 256; ++i) {
            int h = i / 128, r = i % 128, c = r / 32, l = r % 32;
            int byte = ql[64 * h + ((c & 1) ? 32 : 0) + l];
            int low = (c >= 2) ? (byte >> 4) : (byte & 0x0f);
            int high = (qh[32 * h + l] >> (2 * c)) & 3;
            int q = low | (high << 4);
            int s8 = sc[i / 16] < 128 ? (int)sc[i / 16] : (int)sc[i / 16] - 256;  /* two's complement */
            out[b * 256 + i] = dsc * (double)s8 * (double)(q - 32);
        }
    }
}

/* Row r of matrix m (0-based) of a stack of matrices [M][rows][K]. */
static void load_row(int wfmt, const void* base, int64_t m, int64_t rows,
                     int64_t K, int64_t r, double* out) {
    int64_t row = m * rows + r;
    if (wfmt == ORACLE_WFMT_BF16) {
        const uint16_t* p = (const uint16_t*)base + row * K;
        for (int64_t i = 0; i < K; ++i) out[i] = oracle_bf16_to_f64(p[i]);
    } else if (wfmt == ORACLE_ROWS_F16) {
        const uint16_t* p = (const uint16_t*)base + row * K;
        for (int64_t i = 0; i < K; ++i) out[i] = oracle_fp16_to_f64(p[i]);
    } else if (wfmt == ORACLE_WFMT_Q4_0) {
        const uint8_t* p = (const uint8_t*)base + row * (K / 32) * 18;
        q4_0_row(p, K, out);
    } else if (wfmt == ORACLE_WFMT_Q8_0) {
        const uint8_t* p = (const uint8_t*)base + row * (K / 32) * 34;
        q8_0_row(p, K, out);
    } else if (wfmt == ORACLE_WFMT_Q5_0) {
        const uint8_t* p = (const uint8_t*)base + row * (K / 32) * 22;
        q5_0_row(p, K, out);
    } else {
        const uint8_t* p = (const uint8_t*)base + row * (K / 256) * 210;
        q6_k_row(p, K, out);
    }
}

void oracle_dequant_rows(int wfmt, const void* base, int64_t rows, int64_t K,
                         double* out) {
    for (int64_t r = 0; r < rows; ++r) load_row(wfmt, base, 0, rows, K, r, out + r * K);
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Steps 1-4 for one token.  logits may be NULL. */
static void route_token(int d, int E, int k, const double* xt, const float* wr,
                        const float* br, double* logits_out, int32_t* ids,
                        double* w) {
    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)calloc((size_t)E, 1);
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        const float* row = wr + (int64_t)e * d;
        for (int i = 0; i < d; ++i) acc += xt[i] * (double)row[i];
        if (br) acc += (double)br[e];
        l[e] = acc;
    }
    double mx = l[0];
    for (int e = 1; e < E; ++e) if (l[e] > mx) mx = l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) { p[e] = exp(l[e] - mx); z += p[e]; }
    for (int e = 0; e < E; ++e) p[e] /= z;
    double psel = 0.0;
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || l[e] > l[best]) best = e;   /* ties: lower index */
        }
        taken[best] = 1;
        ids[j] = best;
        psel += p[best];
    }
    for (int j = 0; j < k; ++j) w[j] = p[ids[j]] / psel;
    if (logits_out) memcpy(logits_out, l, sizeof(double) * (size_t)E);
    free(l); free(p); free(taken);
}

static void x_row(const uint16_t* x, int d, int t, double* xt) {
    for (int i = 0; i < d; ++i) xt[i] = oracle_bf16_to_f64(x[(int64_t)t * d + i]);
}

int oracle_route(int T, int d, int E, int k, const uint16_t* x, const float* wr,
                 const float* br, double* logits, int32_t* ids, double* w) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || !x || !wr || !ids || !w)
        return 1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        if (!xt) { bad = 1; continue; }
        x_row(x, d, t, xt);
        route_token(d, E, k, xt, wr, br, logits ? logits + (int64_t)t * E : NULL,
                    ids + (int64_t)t * k, w + (int64_t)t * k);
        free(xt);
    }
    return bad ? 2 : 0;
}

/* Step 5: counting sort of the T*k (token, choice) pairs by expert, stable in
 * the pair index p = t*k + j, so tokens are ascending inside each expert. */
int oracle_buckets(int T, int k, int E, const int32_t* ids, int32_t* counts,
                   int32_t* offsets, int32_t* slot_pair) {
    if (T < 0 || k <= 0 || E <= 0 || !ids || !counts || !offsets) return 1;
    int64_t n = (int64_t)T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < n; ++p) {
        if (ids[p] < 0 || ids[p] >= E) return 2;
        counts[ids[p]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    if (slot_pair) {
        int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
        for (int64_t p = 0; p < n; ++p) {
            int e = ids[p];
            slot_pair[offsets[e] + fill[e]] = (int32_t)p;
            fill[e]++;
        }
        free(fill);
    }
    return 0;
}

/* Storage of the gate/up and of the down matrices for a weight format:
 * every format stores all three alike, except BF16_F16DOWN (gate/up bf16,
 * down fp16). */
static int gate_up_fmt(int wfmt) { return wfmt == ORACLE_WFMT_BF16_F16DOWN ? ORACLE_WFMT_BF16 : wfmt; }
static int down_fmt(int wfmt) { return wfmt == ORACLE_WFMT_BF16_F16DOWN ? ORACLE_ROWS_F16 : wfmt; }

/* Step 6 for one token and one expert m of a stack: y = Wd (SiLU(Wg x) * Wu x). */
static void expert_ffn(int wfmt, int d, int Fh, const void* wg, const void* wu,
                       const void* wd, int64_t m, const double* xt, double* y) {
    double* h = (double*)malloc(sizeof(double) * (size_t)Fh);
#pragma omp parallel
    {
        double* row = (double*)malloc(sizeof(double) * (size_t)((d > Fh) ? d : Fh));
#pragma omp for schedule(static)
        for (int f = 0; f < Fh; ++f) {
            double g = 0.0, u = 0.0;
            load_row(gate_up_fmt(wfmt), wg, m, Fh, d, f, row);
            for (int i = 0; i < d; ++i) g += row[i] * xt[i];
            load_row(gate_up_fmt(wfmt), wu, m, Fh, d, f, row);
            for (int i = 0; i < d; ++i) u += row[i] * xt[i];
            h[f] = silu(g) * u;
        }
#pragma omp for schedule(static)
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            load_row(down_fmt(wfmt), wd, m, d, Fh, j, row);
            for (int f = 0; f < Fh; ++f) acc += row[f] * h[f];
            y[j] = acc;
        }
        free(row);
    }
    free(h);
}

/* Steps 1-7 for the tokens listed in `tokens` (NULL: tokens 0..n_tokens-1).
 * out [n_tokens][d]; ids, w [n_tokens][k]; logits [n_tokens][E] (optional).
 * n_threads <= 0 keeps the OpenMP default. */
int oracle_forward(int d, int E, int k, int F, int S, int Fs, int wfmt,
                   const uint16_t* x, int T, const float* wr, const float* br,
                   const void* wg, const void* wu, const void* wd,
                   const void* sg, const void* su, const void* sd,
                   const int32_t* tokens, int n_tokens, double* out,
                   int32_t* ids, double* w, double* logits, int n_threads) {
    if (d <= 0 || E <= 0 || k <= 0 || k > E || F <= 0 || S < 0 || !x || !wr ||
        !wg || !wu || !wd || !out || !ids || !w || n_tokens < 0)
        return 1;
    if (S > 0 && (Fs <= 0 || !sg || !su || !sd)) return 1;
    if (wfmt != ORACLE_WFMT_BF16 && wfmt != ORACLE_WFMT_Q4_0 && wfmt != ORACLE_WFMT_Q8_0 &&
        wfmt != ORACLE_WFMT_Q5_0 && wfmt != ORACLE_WFMT_Q6_K && wfmt != ORACLE_WFMT_BF16_F16DOWN)
        return 1;
    if (wfmt != ORACLE_WFMT_BF16 && wfmt != ORACLE_WFMT_BF16_F16DOWN &&
        (d % 32 || F % 32 || (S > 0 && Fs % 32)))
        return 1;
    if (wfmt == ORACLE_WFMT_Q6_K && (d % 256 || F % 256 || (S > 0 && Fs % 256))) return 1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    double* xt = (double*)malloc(sizeof(double) * (size_t)d);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    for (int n = 0; n < n_tokens; ++n) {
        int t = tokens ? tokens[n] : n;
        if (t < 0 || t >= T) { free(xt); free(y); return 2; }
        x_row(x, d, t, xt);
        int32_t* idn = ids + (int64_t)n * k;
        double* wn = w + (int64_t)n * k;
        route_token(d, E, k, xt, wr, br, logits ? logits + (int64_t)n * E : NULL,
                    idn, wn);
        double* o = out + (int64_t)n * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        for (int j = 0; j < k; ++j) {
            expert_ffn(wfmt, d, F, wg, wu, wd, idn[j], xt, y);
            for (int i = 0; i < d; ++i) o[i] += wn[j] * y[i];
        }
        for (int s = 0; s < S; ++s) {
            expert_ffn(wfmt, d, Fs, sg, su, sd, s, xt, y);
            for (int i = 0; i < d; ++i) o[i] += y[i];
        }
    }
    free(xt);
    free(y);
    return 0;
}

/* Steps 6-7 alone, for routing decided elsewhere: out_t = sum_j w_j
 * FFN_{ids_j}(x_t) + sum_s FFN_s(x_t) for the listed tokens, with the given
 * ids [n_tokens][k] and weights [n_tokens][k] (fp64) in place of steps 1-4.
 * The parity tests use it to check the output of a token whose k-th and
 * (k+1)-th logits nearly tie, where fp32 and fp64 may pick different experts:
 * the GPU's own choice is then evaluated exactly. */
int oracle_forward_routed(int d, int E, int k, int F, int S, int Fs, int wfmt,
                          const uint16_t* x, int T,
                          const void* wg, const void* wu, const void* wd,
                          const void* sg, const void* su, const void* sd,
                          const int32_t* tokens, int n_tokens, const int32_t* ids,
                          const double* w, double* out, int n_threads) {
    if (d <= 0 || E <= 0 || k <= 0 || F <= 0 || S < 0 || !x || !wg || !wu || !wd || !ids ||
        !w || !out || n_tokens < 0)
        return 1;
    if (S > 0 && (Fs <= 0 || !sg || !su || !sd)) return 1;
    if (wfmt != ORACLE_WFMT_BF16 && wfmt != ORACLE_WFMT_Q4_0 && wfmt != ORACLE_WFMT_Q8_0 &&
        wfmt != ORACLE_WFMT_Q5_0 && wfmt != ORACLE_WFMT_Q6_K && wfmt != ORACLE_WFMT_BF16_F16DOWN)
        return 1;
    if (wfmt != ORACLE_WFMT_BF16 && wfmt != ORACLE_WFMT_BF16_F16DOWN &&
        (d % 32 || F % 32 || (S > 0 && Fs % 32)))
        return 1;
    if (wfmt == ORACLE_WFMT_Q6_K && (d % 256 || F % 256 || (S > 0 && Fs % 256))) return 1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    double* xt = (double*)malloc(sizeof(double) * (size_t)d);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    for (int n = 0; n < n_tokens; ++n) {
        int t = tokens ? tokens[n] : n;
        if (t < 0 || t >= T) { free(xt); free(y); return 2; }
        x_row(x, d, t, xt);
        double* o = out + (int64_t)n * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = ids[(int64_t)n * k + j];
            if (e < 0 || e >= E) { free(xt); free(y); return 3; }
            expert_ffn(wfmt, d, F, wg, wu, wd, e, xt, y);
            for (int i = 0; i < d; ++i) o[i] += w[(int64_t)n * k + j] * y[i];
        }
        for (int s2 = 0; s2 < S; ++s2) {
            expert_ffn(wfmt, d, Fs, sg, su, sd, s2, xt, y);
            for (int i = 0; i < d; ++i) o[i] += y[i];
        }
    }
    free(xt);
    free(y);
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
