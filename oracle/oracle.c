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

/* UOS boundary: the abstract fixes the optimal scale boundary at Qmax = 7.25. */
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
 * while P*V uses the quantized ones -- the error in the row-wise normalization that the
 * abstract attributes to plain MXFP4 attention (reading).
 *
 * The softmax loop (the abstract's softmax loop; reading: the standard
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

/* ======================================================================
 * NVFP4 comparison variant.
 *
 * The abstract compares MXAttention with NVFP4 baselines and
 * gives no definition of them.  Reading: NVIDIA's NVFP4 format -- E2M1
 * elements in blocks of 16 with one unsigned E4M3 (OCP FP8 E4M3) scale per
 * block, and a second, per-tensor fp32 scale -- applied to the same four
 * operands and the same softmax loop as the MXFP4 path.  The scale
 * arithmetic runs in fp32 (round to nearest), the precision the GPU path
 * computes it in, so that codes and scales decided from bf16 inputs compare
 * bit for bit.  Readings, each marked below:
 *   - the "tensor" of the second-level scale is one (batch, head) slice of
 *     Q, K or V ([N, d]);
 *   - g = 448 / amax (fp32) maps the slice's largest block to the E4M3
 *     maximum; amax is floored at 2^-100 so g stays finite;
 *   - block scale sb = E4M3(amax_block * g), round to nearest even,
 *     saturating at 448; element factor r = (6 g) / sb (fp32), element code
 *     E2M1(x * r) (x * r in fp32); a block whose scale rounds to 0 is all 0;
 *   - value = code * sb / (6 g);
 *   - P (the unnormalized exponentials, <= 1 by construction) takes g = 448
 *     without a data pass, blocks of 16 keys aligned to key-tile starts;
 *     its block scale is E4M3(fp32(pmax) * 448) and its codes are decided in
 *     fp64 from the exact exponentials, like the MXFP4 path's P.
 * ====================================================================== */

/* OCP FP8 E4M3 ("fn": no infinities, 0x7F is NaN): bias 7, 3 mantissa bits,
 * largest finite 448 = 1.75 * 2^8, subnormals down to 2^-9. */
double oracle_e4m3_decode(uint8_t code) {
    int e = (code >> 3) & 0xF, m = code & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -v : v;
}

/* |v| -> E4M3 code (sign dropped: block scales are non-negative).  Round to
 * nearest, ties to the even code; values at or above 448 saturate to 448
 * (reading: the satfinite conversion NVFP4 scales use). */
uint8_t oracle_e4m3_encode(double v) {
    double a = fabs(v);
    if (!(a < 448.0)) return 0x7E;
    if (a < ldexp(1.0, -6)) { /* subnormal range: steps of 2^-9; 8 * 2^-9 is the smallest normal (code 0x08) */
        double m = nearbyint(ldexp(a, 9));
        return (uint8_t)m;
    }
    int E;
    (void)frexp(a, &E); /* a = f 2^E, f in [0.5, 1): floor(log2 a) = E - 1 */
    int ex = E - 1;
    double q = nearbyint(ldexp(a, 3 - ex)); /* in [8, 16] */
    if (q >= 16.0) {
        q = 8.0;
        ex++;
    }
    int code = ((ex + 7) << 3) | ((int)q - 8);
    return (uint8_t)(code > 0x7E ? 0x7E : code);
}

void oracle_e4m3_encode_batch(const double* v, int64_t n, uint8_t* codes) {
    for (int64_t i = 0; i < n; i++) codes[i] = oracle_e4m3_encode(v[i]);
}

/* Second-level scale of a slice with absolute maximum amax: g = 448 / amax in fp32. */
float oracle_nvfp4_global(double amax) {
    float a = (float)amax;
    const float floor_ = 0x1p-100f;
    if (!(a > floor_)) a = floor_;
    return 448.0f / a;
}

/* One block of n <= 16 fp32-exact values (positions n..15 count as zeros)
 * with second-level scale g: returns the E4M3 scale byte, writes n codes. */
static uint8_t nvfp4_quantize_block(const float* x, int n, float g, uint8_t* codes) {
    float amax = 0.0f;
    for (int i = 0; i < n; i++) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    volatile float prod = amax * g; /* fp32 product, rounded once */
    uint8_t sb = oracle_e4m3_encode((double)prod);
    double sbv = oracle_e4m3_decode(sb);
    if (sbv == 0.0) {
        for (int i = 0; i < n; i++) codes[i] = signbit(x[i]) ? 8u : 0u;
        return sb;
    }
    volatile float G = 6.0f * g;
    volatile float r = G / (float)sbv;
    for (int i = 0; i < n; i++) {
        volatile float v = x[i] * r;
        codes[i] = oracle_e2m1_encode((double)v);
    }
    return sb;
}

/*
 * NVFP4 rows: x bf16 bits [rows, cols], cols % 16 == 0, one second-level
 * scale g for all of them.  codes [rows, cols/2] (element 2i in the low
 * nibble), scales [rows, cols/16] E4M3 bytes.
 */
void oracle_nvfp4_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, float g, uint8_t* codes,
                                uint8_t* scales) {
    float blk[16];
    uint8_t c[16];
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < cols / 16; b++) {
            for (int i = 0; i < 16; i++) blk[i] = (float)oracle_bf16_to_double(x[r * cols + b * 16 + i]);
            scales[r * (cols / 16) + b] = nvfp4_quantize_block(blk, 16, g, c);
            for (int i = 0; i < 8; i++) codes[r * (cols / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
}

/*
 * NVFP4 V^T: v bf16 bits [BH, N, d], g[BH] one scale per (batch, head);
 * blocks of 16 tokens per channel, tokens padded with zeros to
 * Npad = ceil(N/32)*32.  codes [BH, d, Npad/2], scales [BH, d, Npad/16].
 */
void oracle_nvfp4_quantize_cols(const uint16_t* v, int64_t BH, int64_t N, int64_t d, const float* g,
                                uint8_t* codes, uint8_t* scales) {
    int64_t npad = (N + 31) / 32 * 32;
    float blk[16];
    uint8_t c[16];
    for (int64_t bh = 0; bh < BH; bh++)
        for (int64_t ch = 0; ch < d; ch++)
            for (int64_t b = 0; b < npad / 16; b++) {
                for (int i = 0; i < 16; i++) {
                    int64_t t = b * 16 + i;
                    blk[i] = (t < N) ? (float)oracle_bf16_to_double(v[(bh * N + t) * d + ch]) : 0.0f;
                }
                scales[(bh * d + ch) * (npad / 16) + b] = nvfp4_quantize_block(blk, 16, g[bh], c);
                for (int i = 0; i < 8; i++)
                    codes[(bh * d + ch) * (npad / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
            }
}

/* NVFP4 row-layout codes/scales back to values: code * sb / (6 g). */
void oracle_nvfp4_dequantize_rows(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, float g,
                                  double* out) {
    volatile float G = 6.0f * g;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < cols; j++) {
            uint8_t byte = codes[r * (cols / 2) + j / 2];
            uint8_t code = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            out[r * cols + j] = oracle_e2m1_decode(code) * oracle_e4m3_decode(scales[r * (cols / 16) + j / 16]) /
                                (double)G;
        }
}

/* Absolute maximum of n bf16 values. */
double oracle_bf16_amax(const uint16_t* x, int64_t n) {
    double m = 0.0;
    for (int64_t i = 0; i < n; i++) {
        double a = fabs(oracle_bf16_to_double(x[i]));
        if (a > m) m = a;
    }
    return m;
}

/*
 * One head of NVFP4 attention: the MXFP4 loop of oracle_attention_head_q
 * with every operand in NVFP4 (see the block comment above).  quant = 0
 * keeps all four operands exact (then this is plain online softmax);
 * p_quant = 0 keeps only P exact.  pnq as in the MXFP4 loop.
 */
int oracle_nvfp4_attention_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t N, int64_t d,
                                int64_t kv_tile, int quant, int p_quant, int pnq, double scale, const int64_t* rows,
                                int64_t nrows, double* O, int nthreads) {
    if (N < 1 || d % 16 != 0 || kv_tile % 32 != 0 || kv_tile < 32) return 1;
    int64_t npad = (N + 31) / 32 * 32;
    double* qd = (double*)malloc(sizeof(double) * (size_t)(N * d));
    double* kd = (double*)malloc(sizeof(double) * (size_t)(N * d));
    double* vt = (double*)malloc(sizeof(double) * (size_t)(d * npad));
    uint8_t* c = (uint8_t*)malloc((size_t)(d * npad / 2 + N * d / 2));
    uint8_t* s = (uint8_t*)malloc((size_t)(d * npad / 16 + N * d / 16));
    if (!qd || !kd || !vt || !c || !s) {
        free(qd), free(kd), free(vt), free(c), free(s);
        return 2;
    }
    if (!quant) {
        for (int64_t j = 0; j < N * d; j++) qd[j] = oracle_bf16_to_double(Q[j]);
        for (int64_t j = 0; j < N * d; j++) kd[j] = oracle_bf16_to_double(K[j]);
        for (int64_t ch = 0; ch < d; ch++)
            for (int64_t t = 0; t < npad; t++) vt[ch * npad + t] = (t < N) ? oracle_bf16_to_double(V[t * d + ch]) : 0.0;
    } else {
        float gq = oracle_nvfp4_global(oracle_bf16_amax(Q, N * d));
        float gk = oracle_nvfp4_global(oracle_bf16_amax(K, N * d));
        float gv = oracle_nvfp4_global(oracle_bf16_amax(V, N * d));
        oracle_nvfp4_quantize_rows(Q, N, d, gq, c, s);
        oracle_nvfp4_dequantize_rows(c, s, N, d, gq, qd);
        oracle_nvfp4_quantize_rows(K, N, d, gk, c, s);
        oracle_nvfp4_dequantize_rows(c, s, N, d, gk, kd);
        oracle_nvfp4_quantize_cols(V, 1, N, d, &gv, c, s);
        oracle_nvfp4_dequantize_rows(c, s, d, npad, gv, vt);
    }
    free(c);
    free(s);
    const int do_p = quant && p_quant;
    int status = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t r = 0; r < nrows; r++) {
        int64_t i = rows[r];
        double* sc = (double*)malloc(sizeof(double) * (size_t)N);
        double* o = (double*)calloc((size_t)d, sizeof(double));
        double* to = (double*)malloc(sizeof(double) * (size_t)d);
        if (!sc || !o || !to || i < 0 || i >= N) {
            status = 3;
            free(sc), free(o), free(to);
            continue;
        }
        for (int64_t j = 0; j < N; j++) {
            double acc = 0.0;
            for (int64_t ch = 0; ch < d; ch++) acc += qd[i * d + ch] * kd[j * d + ch];
            sc[j] = acc * scale;
        }
        double m = -INFINITY, l = 0.0;
        for (int64_t t0 = 0; t0 < N; t0 += kv_tile) {
            int64_t t1 = t0 + kv_tile < N ? t0 + kv_tile : N;
            double tile_max = -INFINITY;
            for (int64_t j = t0; j < t1; j++)
                if (sc[j] > tile_max) tile_max = sc[j];
            double m_new = m > tile_max ? m : tile_max;
            double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
            double sum_p = 0.0, sum_q = 0.0;
            for (int64_t ch = 0; ch < d; ch++) to[ch] = 0.0;
            for (int64_t b0 = t0; b0 < t0 + kv_tile; b0 += 16) {
                double p[16], q[16];
                double pmax = 0.0;
                for (int k = 0; k < 16; k++) {
                    int64_t j = b0 + k;
                    p[k] = (j < t1) ? exp(sc[j] - m_new) : 0.0;
                    if (p[k] > pmax) pmax = p[k];
                }
                if (!do_p) {
                    for (int k = 0; k < 16; k++) q[k] = p[k];
                } else {
                    volatile float prod = (float)pmax * 448.0f;
                    uint8_t sb = oracle_e4m3_encode((double)prod);
                    double sbv = oracle_e4m3_decode(sb);
                    if (sbv == 0.0) {
                        for (int k = 0; k < 16; k++) q[k] = 0.0;
                    } else {
                        volatile float rr = 2688.0f / (float)sbv;
                        for (int k = 0; k < 16; k++)
                            q[k] = oracle_e2m1_decode(oracle_e2m1_encode(p[k] * (double)rr)) * sbv / 2688.0;
                    }
                }
                for (int k = 0; k < 16; k++) {
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
        free(sc), free(o), free(to);
    }
    free(qd);
    free(kd);
    free(vt);
    return status;
}
