/*
 * oracle.c -- plain, slow, fp64 CPU reference for MXFP4 attention with
 * Universal Optimal Scaling (UOS) and Pre-Normalization Quantization (PNQ).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * Source: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
 * Quantization for MXFP4 Attention", abstract (the only passage the pages give
 * on the method).  The abstract fixes: MXFP4 operands with power-of-two
 * microscaling, the UOS scaling boundary Qmax = 7.25, and PNQ, which quantizes
 * the unnormalized softmax exponentials before the row-wise sum.  Everything
 * else below is a reading, marked "reading:":
 *   - MXFP4 = the OCP Microscaling (MX) format that the abstract's "OCP
 *     MXFP4" names: 32-element blocks, E2M1 elements {0,.5,1,1.5,2,3,4,6}
 *     with a sign bit, one E8M0 power-of-two scale per block.
 *   - OCP scale rule: e = floor(log2 amax) - 2 (2 = largest E2M1 exponent).
 *   - UOS scale rule: the smallest integer e with amax <= 7.25 * 2^e.
 *   - the same boundary rule for any Qmax in (4, 8) (the abstract names the
 *     boundary Qmax; 7.25 is its choice), used to sweep the boundary; OCP is
 *     the limit Qmax -> 8 from below (reading).
 *   - elements: round to nearest, ties to the even code, saturate at 6.
 *
 * Every loop follows the definitions in the order the method states them;
 * no blocking, fusion or reordering.  Floating point is fp64 throughout.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_RULE_OCP 0
#define ORACLE_RULE_UOS 1
#define ORACLE_RULE_NONE 2 /* identity: no quantization at all */
#define ORACLE_RULE_QMAX 3 /* boundary rule with a caller-chosen Qmax in (4, 8) */

/* E2M1 magnitudes in code order (code bits: sign | exponent(2) | mantissa(1)). */
static const double kE2M1Magnitude[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* UOS boundary, from the abstract: "optimal scaling boundary Qmax=7.25". */
static const double kUosQmax = 7.25;

/* bfloat16 bit pattern -> value: the top 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E2M1 code -> value (OCP MX element format). */
double oracle_e2m1_decode(uint8_t code) {
    double m = kE2M1Magnitude[code & 7u];
    return (code & 8u) ? -m : m;
}

/*
 * Value -> E2M1 code: nearest representable magnitude, ties to the even code
 * (reading: round-to-nearest-even, as for IEEE formats), magnitudes >= 6
 * saturate to 6 (reading: MX conversions saturate).  The sign bit is kept even
 * when the magnitude rounds to zero, so -0 encodes as 0x8 (reading).
 */
uint8_t oracle_e2m1_encode(double v) {
    uint8_t sign = signbit(v) ? 8u : 0u;
    double a = fabs(v);
    if (a >= kE2M1Magnitude[7]) return (uint8_t)(sign | 7u);
    int lo = 0;
    while (!(a < kE2M1Magnitude[lo + 1])) lo++;
    double d_lo = a - kE2M1Magnitude[lo];
    double d_hi = kE2M1Magnitude[lo + 1] - a;
    int idx;
    if (d_lo < d_hi)
        idx = lo;
    else if (d_hi < d_lo)
        idx = lo + 1;
    else
        idx = (lo % 2 == 0) ? lo : lo + 1; /* tie: the even code */
    return (uint8_t)(sign | (uint8_t)idx);
}

void oracle_e2m1_encode_batch(const double* v, int64_t n, uint8_t* codes) {
    for (int64_t i = 0; i < n; i++) codes[i] = oracle_e2m1_encode(v[i]);
}

/*
 * Shared block exponent e (scale 2^e) from the block's absolute maximum.
 *   OCP (the baseline the abstract compares against): e = floor(log2 amax) - 2.
 *   UOS (abstract: data-free boundary Qmax = 7.25): smallest e with
 *       amax <= Qmax * 2^e, so amax / 2^e lies in (Qmax/2, Qmax]; values in
 *       (6, Qmax] then saturate to 6.
 *   QMAX: the same boundary rule with the caller's Qmax (reading: any
 *       boundary in (4, 8) is a valid member of the family UOS picks from).
 * Reading for the cases the pages leave open: amax == 0 (or not > 0) gives
 * e = -127; e is clamped to the E8M0 range [-127, 127].
 */
static int scale_exponent(double amax, int rule, double qmax) {
    if (!(amax > 0.0)) return -127;
    int E;
    (void)frexp(amax, &E); /* amax = f * 2^E, f in [0.5, 1)  =>  floor(log2 amax) = E - 1 */
    int floor_log2 = E - 1;
    int e;
    if (rule == ORACLE_RULE_OCP) {
        e = floor_log2 - 2;
    } else {
        double q = (rule == ORACLE_RULE_UOS) ? kUosQmax : qmax;
        e = floor_log2 - 4; /* q * 2^(floor_log2 - 4) < amax for q < 16: the search starts below the answer */
        while (amax > q * ldexp(1.0, e)) e++;
    }
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

int oracle_scale_exponent(double amax, int rule) { return scale_exponent(amax, rule, kUosQmax); }

void oracle_scale_exponent_batch(const double* amax, int64_t n, int rule, int32_t* e) {
    for (int64_t i = 0; i < n; i++) e[i] = scale_exponent(amax[i], rule, kUosQmax);
}

void oracle_scale_exponent_q_batch(const double* amax, int64_t n, int rule, double qmax, int32_t* e) {
    for (int64_t i = 0; i < n; i++) e[i] = scale_exponent(amax[i], rule, qmax);
}

/* Quantize one block of n values (n <= 32; positions n..31 count as zeros).
 * Returns e; writes n codes.  */
static int quantize_block(const double* x, int n, int rule, double qmax, uint8_t* codes) {
    double amax = 0.0;
    for (int i = 0; i < n; i++) {
        double a = fabs(x[i]);
        if (a > amax) amax = a;
    }
    int e = scale_exponent(amax, rule, qmax);
    for (int i = 0; i < n; i++) codes[i] = oracle_e2m1_encode(ldexp(x[i], -e));
    return e;
}

/*
 * Row quantization (Q and K: blocks of 32 along the head dimension d; also the
 * standalone quantize op).  x: bf16 bits [rows, cols], cols % 32 == 0.
 * codes: [rows, cols/2] bytes, element 2i in the low nibble, 2i+1 in the high
 * nibble.  scales: [rows, cols/32] E8M0 bytes (e + 127).
 */
void oracle_quantize_rows_q(const uint16_t* x, int64_t rows, int64_t cols, int rule, double qmax,
                            uint8_t* codes, uint8_t* scales) {
    double blk[32];
    uint8_t c[32];
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < cols / 32; b++) {
            for (int i = 0; i < 32; i++) blk[i] = oracle_bf16_to_double(x[r * cols + b * 32 + i]);
            int e = quantize_block(blk, 32, rule, qmax, c);
            scales[r * (cols / 32) + b] = (uint8_t)(e + 127);
            for (int i = 0; i < 16; i++)
                codes[r * (cols / 2) + b * 16 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
}

void oracle_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, int rule, uint8_t* codes,
                          uint8_t* scales) {
    oracle_quantize_rows_q(x, rows, cols, rule, kUosQmax, codes, scales);
}

/*
 * Column quantization of V (reading: the MX scale runs along the contraction
 * dimension of each product, which for P*V is the token axis).
 * v: bf16 bits [BH, N, d].  Output is V transposed: codes [BH, d, Npad/2],
 * scales [BH, d, Npad/32], Npad = ceil(N/32)*32, tokens >= N count as zeros.
 */
void oracle_quantize_cols_q(const uint16_t* v, int64_t BH, int64_t N, int64_t d, int rule, double qmax,
                            uint8_t* codes, uint8_t* scales) {
    int64_t npad = (N + 31) / 32 * 32;
    double blk[32];
    uint8_t c[32];
    for (int64_t bh = 0; bh < BH; bh++) {
        for (int64_t ch = 0; ch < d; ch++) {
            for (int64_t b = 0; b < npad / 32; b++) {
                for (int i = 0; i < 32; i++) {
                    int64_t t = b * 32 + i;
                    blk[i] = (t < N) ? oracle_bf16_to_double(v[(bh * N + t) * d + ch]) : 0.0;
                }
                int e = quantize_block(blk, 32, rule, qmax, c);
                scales[(bh * d + ch) * (npad / 32) + b] = (uint8_t)(e + 127);
                for (int i = 0; i < 16; i++)
                    codes[(bh * d + ch) * (npad / 2) + b * 16 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
            }
        }
    }
}

void oracle_quantize_cols(const uint16_t* v, int64_t BH, int64_t N, int64_t d, int rule, uint8_t* codes,
                          uint8_t* scales) {
    oracle_quantize_cols_q(v, BH, N, d, rule, kUosQmax, codes, scales);
}

/* Dequantize row-layout codes/scales back to values. */
void oracle_dequantize_rows(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                            double* out) {
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < cols; j++) {
            uint8_t byte = codes[r * (cols / 2) + j / 2];
            uint8_t code = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            int e = (int)scales[r * (cols / 32) + j / 32] - 127;
            out[r * cols + j] = ldexp(oracle_e2m1_decode(code), e);
        }
}

/*
 * One head of MXFP4 attention, for a chosen subset of query rows.
 *
 * Q, K, V: bf16 bits [N, d] of one (batch, head).  in_rule quantizes Q, K
 * (blocks along d) and V (blocks along tokens) -- ORACLE_RULE_NONE keeps the
 * bf16 values.  p_rule quantizes the exponentials P (blocks of 32 along the
 * key axis, aligned to tile starts) -- ORACLE_RULE_NONE keeps them exact.
 * pnq = 1: PNQ (abstract: quantize the unnormalized exponentials before the
 * row-wise summation, so the row sum is built from the same quantized values
 * that weight V).  pnq = 0: the row sum uses the unquantized exponentials
 * while P*V uses the quantized ones -- the "row-wise normalization error" the
 * abstract attributes to plain MXFP4 attention (reading).
 *
 * The softmax loop (abstract: "the softmax loop"; reading: the standard
 * online softmax over key tiles of kv_tile columns, ascending), per row i:
 *   s_j   = (deq(Q_i) . deq(K_j)) * scale      (scale applied after quantization: reading)
 *   m = -inf, l = 0, o = 0
 *   for each tile:
 *     m_new = max(m, max_j s_j)
 *     alpha = exp(m - m_new)   (0 on the first tile)
 *     p_j   = exp(s_j - m_new)  (0 beyond N)      -- the running max after this tile: reading
 *     q_j   = deq(quantize(p_j per 32-column block))
 *     l = alpha*l + (pnq ? sum q_j : sum p_j)
 *     o = alpha*o + sum q_j * deq(V_j)
 *     m = m_new
 *   O_i = o / l
 *
 * qmax: the boundary of ORACLE_RULE_QMAX (both rules; ignored by the others).
 * rows: indices of the query rows to compute; O: [nrows, d] fp64.
 */
int oracle_attention_head_q(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t N, int64_t d,
                            int64_t kv_tile, int in_rule, int p_rule, double qmax, int pnq, double scale,
                            const int64_t* rows, int64_t nrows, double* O, int nthreads) {
    if (N < 1 || d % 32 != 0 || kv_tile % 32 != 0 || kv_tile < 32) return 1;
    int64_t npad = (N + 31) / 32 * 32;
    double* kd = (double*)malloc(sizeof(double) * (size_t)(N * d));
    double* vt = (double*)malloc(sizeof(double) * (size_t)(d * npad)); /* V^T values [d, npad] */
    if (!kd || !vt) {
        free(kd);
        free(vt);
        return 2;
    }
    /* K (blocks along d) */
    if (in_rule == ORACLE_RULE_NONE) {
        for (int64_t j = 0; j < N * d; j++) kd[j] = oracle_bf16_to_double(K[j]);
    } else {
        uint8_t* c = (uint8_t*)malloc((size_t)(N * d / 2));
        uint8_t* s = (uint8_t*)malloc((size_t)(N * d / 32));
        oracle_quantize_rows_q(K, N, d, in_rule, qmax, c, s);
        oracle_dequantize_rows(c, s, N, d, kd);
        free(c);
        free(s);
    }
    /* V (blocks along tokens), kept transposed */
    if (in_rule == ORACLE_RULE_NONE) {
        for (int64_t ch = 0; ch < d; ch++)
            for (int64_t t = 0; t < npad; t++)
                vt[ch * npad + t] = (t < N) ? oracle_bf16_to_double(V[t * d + ch]) : 0.0;
    } else {
        uint8_t* c = (uint8_t*)malloc((size_t)(d * npad / 2));
        uint8_t* s = (uint8_t*)malloc((size_t)(d * npad / 32));
        oracle_quantize_cols_q(V, 1, N, d, in_rule, qmax, c, s);
        oracle_dequantize_rows(c, s, d, npad, vt);
        free(c);
        free(s);
    }

    int status = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t r = 0; r < nrows; r++) {
        int64_t i = rows[r];
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* qd = (double*)malloc(sizeof(double) * (size_t)d);
        double* o = (double*)calloc((size_t)d, sizeof(double));
        double* to = (double*)malloc(sizeof(double) * (size_t)d);
        if (!s || !qd || !o || !to || i < 0 || i >= N) {
            status = 3;
            free(s), free(qd), free(o), free(to);
            continue;
        }
        /* deq(Q_i) */
        if (in_rule == ORACLE_RULE_NONE) {
            for (int64_t ch = 0; ch < d; ch++) qd[ch] = oracle_bf16_to_double(Q[i * d + ch]);
        } else {
            uint8_t c[64], sc[4];
            oracle_quantize_rows_q(Q + i * d, 1, d, in_rule, qmax, c, sc);
            oracle_dequantize_rows(c, sc, 1, d, qd);
        }
        /* s_j */
        for (int64_t j = 0; j < N; j++) {
            double acc = 0.0;
            for (int64_t ch = 0; ch < d; ch++) acc += qd[ch] * kd[j * d + ch];
            s[j] = acc * scale;
        }
        /* the softmax loop over key tiles, ascending */
        double m = -INFINITY, l = 0.0;
        for (int64_t t0 = 0; t0 < N; t0 += kv_tile) {
            int64_t t1 = t0 + kv_tile < N ? t0 + kv_tile : N;
            double tile_max = -INFINITY;
            for (int64_t j = t0; j < t1; j++)
                if (s[j] > tile_max) tile_max = s[j];
            double m_new = m > tile_max ? m : tile_max;
            double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
            double sum_p = 0.0, sum_q = 0.0;
            for (int64_t ch = 0; ch < d; ch++) to[ch] = 0.0;
            for (int64_t b0 = t0; b0 < t0 + kv_tile; b0 += 32) {
                double p[32], q[32];
                uint8_t c[32];
                for (int k = 0; k < 32; k++) {
                    int64_t j = b0 + k;
                    p[k] = (j < t1) ? exp(s[j] - m_new) : 0.0;
                }
                if (p_rule == ORACLE_RULE_NONE) {
                    for (int k = 0; k < 32; k++) q[k] = p[k];
                } else {
                    int e = quantize_block(p, 32, p_rule, qmax, c);
                    for (int k = 0; k < 32; k++) q[k] = ldexp(oracle_e2m1_decode(c[k]), e);
                }
                for (int k = 0; k < 32; k++) {
                    int64_t j = b0 + k;
                    if (j >= t1) continue;
                    sum_p += p[k];
                    sum_q += q[k];
                    for (int64_t ch = 0; ch < d; ch++) to[ch] += q[k] * vt[ch * npad + j];
                }
            }
            l = alpha * l + (pnq ? sum_q : sum_p);
            for (int64_t ch = 0; ch < d; ch++) o[ch] = alpha * o[ch] + to[ch];
            m = m_new;
        }
        for (int64_t ch = 0; ch < d; ch++) O[r * d + ch] = o[ch] / l;
        free(s), free(qd), free(o), free(to);
    }
    free(kd);
    free(vt);
    return status;
}

int oracle_attention_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t N, int64_t d,
                          int64_t kv_tile, int in_rule, int p_rule, int pnq, double scale, const int64_t* rows,
                          int64_t nrows, double* O, int nthreads) {
    return oracle_attention_head_q(Q, K, V, N, d, kv_tile, in_rule, p_rule, kUosQmax, pnq, scale, rows, nrows, O,
                                   nthreads);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
