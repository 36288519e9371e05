/*
 * nvfp4moe oracle: TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, single-purpose CPU implementation of what the NVFP4 MoE
 * expert-layer path computes. Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library. It shares no code,
 * header, table or constant with the CUDA library, and it never receives an
 * input that the CUDA library produced.
 *
 * Sources. The method is the one described in the write-ups of Thinking
 * Machines Lab's "End-to-End 4-Bit Training" post:
 *   [P1] news.t0001.com, "Thinking Machines 详解 Inkling 2 Small 原生 4-bit
 *        前向训练完整流程", list "训练数值格式分工清单" (NVFP4 expert forward,
 *        MXFP8 backward with stochastic rounding, quantized cross-GPU traffic).
 *   [P2] aicoder.com, "Thinking Machines Details End-to-End 4-Bit Training for
 *        Inkling 2 Small", sections "Key Takeaways", "Background" (NVFP4 uses
 *        about 4.5 bits per value) and "Architecture highlights" (MXFP8 backward
 *        with re-quantization and stochastic rounding; 32-dimensional random
 *        Hadamard transform before quantizing the combine traffic; the kernel
 *        stack is fully deterministic).
 *   [P4] 10100.com, "Inkling 2 Small", "PART 01" (384 experts, top-8, 48 layers).
 * None of the pages prints a formula. Every numeric rule below is a reading,
 * marked READING at the place it is applied.
 *
 * Precision. Where a floating-point value decides an integer (a quantized
 * code, a scale code, a top-k index) the oracle takes that decision in IEEE
 * fp32 with round-to-nearest and no contraction, the precision the kernels
 * use. Everything else (dequantized products, GEMMs, SwiGLU, softmax, combine)
 * is fp64. Build with -ffp-contract=off.
 *
 * Codecs are brute force on purpose: nearest value by exhaustive search over
 * the format's code table, not bit manipulation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define ORACLE_API __attribute__((visibility("default")))

/* Threads of the parallel loops (the rows of oracle_gemm_f64). No result
 * depends on it: the rows are independent and each is summed in order. */
ORACLE_API void oracle_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
ORACLE_API int oracle_max_threads(void) { return omp_get_max_threads(); }

/* ------------------------------------------------------------------------ */
/* bf16                                                                      */
/* ------------------------------------------------------------------------ */

ORACLE_API float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to the nearest bf16 value, ties to even (8 significant bits,
 * exponent range of fp32). Written from the definition: pick the quantum of
 * the binade of |v|, round |v|/quantum to an integer with ties to even. */
ORACLE_API uint16_t oracle_bf16_from_f64(double v) {
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else {
        int e;
        frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1) -> floor(log2 a) = e - 1 */
        int eb = e - 1;
        if (eb < -126) eb = -126; /* subnormal bf16 quantum is 2^-133 */
        double quantum = ldexp(1.0, eb - 7);
        double q = a / quantum;   /* exact: division by a power of two */
        double n = nearbyint(q);  /* default rounding mode: ties to even */
        r = n * quantum;
        if (r > 3.3895313892515355e38) r = INFINITY; /* beyond max bf16 */
    }
    float f = (float)r; /* exact: r has at most 8 significant bits */
    if (signbit(v)) f = -f;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (4-bit float): sign bit 3, magnitude code 0..7                        */
/* ------------------------------------------------------------------------ */

/* READING: the eight E2M1 magnitudes of the NVFP4 element format. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

ORACLE_API double oracle_e2m1_decode(uint8_t nib) {
    double m = E2M1_MAG[nib & 7];
    return (nib & 8) ? -m : m;
}

/* Nearest magnitude on the grid; on a tie the even code wins; beyond 6 the
 * nearest point is 6 (saturation). The sign bit is the sign of the input, so
 * negative values that round to zero give the code 0x8. */
ORACLE_API uint8_t oracle_e2m1_encode(float v) {
    double a = fabs((double)v);
    if (a > 6.0) a = 6.0; /* saturation; also keeps the distances below exact */
    int best = 0;
    double bd = INFINITY;
    for (int m = 0; m < 8; ++m) {
        double d = fabs(a - E2M1_MAG[m]);
        if (d < bd || (d == bd && (m % 2) == 0)) {
            bd = d;
            best = m;
        }
    }
    return (uint8_t)((signbit(v) ? 8 : 0) | best);
}

/* ------------------------------------------------------------------------ */
/* E4M3 (OCP FN): bias 7, no infinities, S.1111.111 is NaN, max 448           */
/* ------------------------------------------------------------------------ */

ORACLE_API double oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round to nearest E4M3 value (ties to the even code), saturating at 448. */
ORACLE_API uint8_t oracle_e4m3_encode(float v) {
    double a = fabs((double)v);
    if (a > 448.0) a = 448.0; /* saturation; also keeps the distances below exact */
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 126; ++c) {
        double d = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (d < bd || (d == bd && (c % 2) == 0)) {
            bd = d;
            best = c;
        }
    }
    return (uint8_t)((signbit(v) ? 0x80 : 0) | best);
}

ORACLE_API double oracle_e8m0_decode(uint8_t c) {
    if (c == 255) return NAN;
    return ldexp(1.0, (int)c - 127);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 quantize / dequantize                                               */
/* ------------------------------------------------------------------------ */
/*
 * NVFP4 ([P2] "Background": about 4.5 bits per value; [P1] "训练数值格式分工清单":
 * the expert forward runs in NVFP4).
 * READING (two-level scaling): one fp32 tensor amax; encode scale
 * S_enc = 2688 / amax (2688 = 6 * 448, the largest E2M1 magnitude times the
 * largest E4M3 value); per 16-element block an E4M3 scale s_b =
 * RNE((amax_b / 6) * S_enc); element codes RNE(x * S_enc / s_b). The stored
 * fp32 decode scale is ts = amax / 2688. A tensor whose amax is 0 (or not
 * finite) uses S_enc = ts = 1. A block whose scale rounds to 0 has all-zero
 * codes. All of this in fp32, one rounding per operation.
 */
static float amax_f32(const float *x, int64_t n) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    return m;
}

static float nvfp4_senc(float amax) {
    return (amax > 0.0f && isfinite(amax)) ? 2688.0f / amax : 1.0f;
}
static float nvfp4_ts(float amax) {
    return (amax > 0.0f && isfinite(amax)) ? amax / 2688.0f : 1.0f;
}

/* Quantize one row of cols values (cols % 16 == 0) given S_enc.
 * codes: cols/2 bytes, element 2i in the low nibble of byte i.
 * scales: cols/16 E4M3 codes. */
static void nvfp4_quantize_row(const float *x, int64_t cols, float S_enc,
                               uint8_t *codes, uint8_t *scales) {
    for (int64_t b = 0; b < cols / 16; ++b) {
        const float *xb = x + b * 16;
        float amax_b = amax_f32(xb, 16);
        float t = amax_b / 6.0f;
        t = t * S_enc;
        uint8_t sc = oracle_e4m3_encode(t);
        float sf = (float)oracle_e4m3_decode(sc);
        float enc = (sf == 0.0f) ? 0.0f : S_enc / sf;
        scales[b] = sc;
        for (int i = 0; i < 16; i += 2) {
            float v0 = xb[i] * enc;
            float v1 = xb[i + 1] * enc;
            uint8_t q0 = oracle_e2m1_encode(v0);
            uint8_t q1 = oracle_e2m1_encode(v1);
            codes[(b * 16 + i) / 2] = (uint8_t)(q0 | (q1 << 4));
        }
    }
}

ORACLE_API float oracle_amax(const float *x, int64_t n) { return amax_f32(x, n); }

/* x: rows x cols fp32 values (bf16 inputs are passed exactly widened).
 * amax_in: NULL to compute max|x| over the whole tensor. */
ORACLE_API void oracle_nvfp4_quantize(const float *x, int64_t rows, int64_t cols,
                                      const float *amax_in, uint8_t *codes,
                                      uint8_t *scales, float *ts_out) {
    float amax = amax_in ? *amax_in : amax_f32(x, rows * cols);
    float S_enc = nvfp4_senc(amax);
    *ts_out = nvfp4_ts(amax);
    for (int64_t r = 0; r < rows; ++r)
        nvfp4_quantize_row(x + r * cols, cols, S_enc, codes + r * (cols / 2),
                           scales + r * (cols / 16));
}

/* x_hat = e2m1(q) * s_b * ts, in fp32 (the first product is exact). */
ORACLE_API void oracle_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales,
                                        float ts, int64_t rows, int64_t cols,
                                        float *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
            float sf = (float)oracle_e4m3_decode(scales[r * (cols / 16) + c / 16]);
            float a = (float)oracle_e2m1_decode(nib) * sf;
            out[r * cols + c] = a * ts;
        }
}

/* Dequantize to fp64 (used by the GEMM reference). */
static double nvfp4_value(const uint8_t *codes, const uint8_t *scales, float ts,
                          int64_t cols, int64_t r, int64_t c) {
    uint8_t byte = codes[r * (cols / 2) + c / 2];
    uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
    return oracle_e2m1_decode(nib) * oracle_e4m3_decode(scales[r * (cols / 16) + c / 16]) *
           (double)ts;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As   */
/* Easy as 1, 2, 3", SC'11), with the round multipliers and Weyl key         */
/* increments published there.                                               */
/* ------------------------------------------------------------------------ */

ORACLE_API void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                                     uint32_t out[4]) {
    uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint32_t k[2] = {key_in[0], key_in[1]};
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c[1] ^ k[0];
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c[3] ^ k[1];
        uint32_t n3 = lo0;
        c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
    }
    memcpy(out, c, 16);
}

/* The random word for logical element i under (seed, offset): key = seed,
 * counter = (i / 4, offset), word i % 4. */
ORACLE_API uint32_t oracle_philox_word(uint64_t seed, uint64_t offset, uint64_t i) {
    uint64_t blk = i >> 2;
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)offset,
                       (uint32_t)(offset >> 32)};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[i & 3];
}

/* ------------------------------------------------------------------------ */
/* MXFP8: E4M3 codes, one E8M0 (power-of-two) scale per 32 elements          */
/* ------------------------------------------------------------------------ */
/*
 * [P1] "训练数值格式分工清单" and [P2] "Key Takeaways": the backward pass uses MXFP8
 * with stochastic rounding to limit gradient bias.
 * READING (scale): the smallest k in [-127, 127] with amax_b <= 448 * 2^k, so
 * no element clips (clipping would bias stochastic rounding); code k + 127.
 * READING (stochastic rounding): with lo <= |v| <= hi the neighbouring E4M3
 * values, round up iff r * 2^-24 < (|v| - lo) / (hi - lo), r the top 24 bits of
 * the element's Philox word. Round-to-nearest-even is the other mode.
 */
static int mx_scale_exp(float amax_b) {
    for (int k = -127; k <= 127; ++k)
        if ((double)amax_b <= 448.0 * ldexp(1.0, k)) return k;
    return 127;
}

static uint8_t e4m3_sr(double v, uint32_t word) {
    double a = fabs(v);
    double lo = 0.0, hi = 448.0;
    for (int c = 0; c <= 126; ++c) {
        double g = oracle_e4m3_decode((uint8_t)c);
        if (g <= a && g > lo) lo = g;
        if (g >= a && g < hi) hi = g;
    }
    double mag = lo;
    if (hi > lo) {
        double r = (double)(word >> 8);
        /* r * 2^-24 < (a - lo) / (hi - lo), compared without division */
        if (r * (hi - lo) < (a - lo) * 16777216.0) mag = hi;
    }
    int code = 0;
    for (int c = 0; c <= 126; ++c)
        if (oracle_e4m3_decode((uint8_t)c) == mag) { code = c; break; }
    return (uint8_t)((signbit(v) ? 0x80 : 0) | code);
}

/* Quantize one 32-block given by 32 values and their logical source indices. */
static void mx_block(const float *vals, const uint64_t *idx, int rounding, uint64_t seed,
                     uint64_t offset, uint8_t *codes_out, int64_t code_stride,
                     uint8_t *scale_out) {
    float amax_b = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float a = fabsf(vals[i]);
        if (a > amax_b) amax_b = a;
    }
    int k = mx_scale_exp(amax_b);
    *scale_out = (uint8_t)(k + 127);
    for (int i = 0; i < 32; ++i) {
        double v = ldexp((double)vals[i], -k); /* exact */
        uint8_t q;
        if (rounding == 1)
            q = e4m3_sr(v, oracle_philox_word(seed, offset, idx[i]));
        else
            q = oracle_e4m3_encode((float)v); /* v is exact in fp32 */
        codes_out[i * code_stride] = q;
    }
}

/*
 * x: rows x cols fp32 values (widened bf16), row-major. Row r of x is row
 * row0 + r of the source tensor, so the logical element index the stochastic
 * draws follow is i = (row0 + r) * cols + c (row0 = 0 for a whole tensor;
 * a larger row0 quantizes a slice of rows with the draws of the whole).
 * axis 0: blocks of 32 along cols. codes [rows x cols], scales [rows x cols/32].
 * axis 1: blocks of 32 along rows inside segments seg_off[0..nseg] (NULL: one
 *   segment of all rows; offsets count rows of x); each segment is
 *   zero-padded to a multiple of 32.
 *   Output is transposed: codes [cols x Rpad], scales [cols x Rpad/32], where
 *   Rpad is the sum of the padded segment lengths.
 * rounding: 0 = round-to-nearest-even, 1 = stochastic.
 */
ORACLE_API void oracle_mxfp8_quantize_at(const float *x, int64_t rows, int64_t cols, int64_t row0,
                                         int axis, const int32_t *seg_off, int32_t nseg,
                                         uint64_t seed, uint64_t offset, int rounding,
                                         uint8_t *codes, uint8_t *scales) {
    float vals[32];
    uint64_t idx[32];
    if (axis == 0) {
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t b = 0; b < cols / 32; ++b) {
                for (int i = 0; i < 32; ++i) {
                    vals[i] = x[r * cols + b * 32 + i];
                    idx[i] = (uint64_t)((row0 + r) * cols + b * 32 + i);
                }
                mx_block(vals, idx, rounding, seed, offset, codes + r * cols + b * 32, 1,
                         scales + r * (cols / 32) + b);
            }
        return;
    }
    int32_t one_seg[2] = {0, (int32_t)rows};
    if (!seg_off) { seg_off = one_seg; nseg = 1; }
    int64_t Rpad = 0;
    for (int s = 0; s < nseg; ++s) Rpad += ((int64_t)(seg_off[s + 1] - seg_off[s]) + 31) / 32 * 32;
    int64_t out_r = 0;
    for (int s = 0; s < nseg; ++s) {
        int64_t r0 = seg_off[s], r1 = seg_off[s + 1];
        int64_t len = (r1 - r0 + 31) / 32 * 32;
        for (int64_t b = 0; b < len / 32; ++b) {
            for (int64_t c = 0; c < cols; ++c) {
                for (int i = 0; i < 32; ++i) {
                    int64_t r = r0 + b * 32 + i;
                    vals[i] = (r < r1) ? x[r * cols + c] : 0.0f;
                    idx[i] = (r < r1) ? (uint64_t)((row0 + r) * cols + c) : 0;
                }
                mx_block(vals, idx, rounding, seed, offset, codes + c * Rpad + out_r + b * 32, 1,
                         scales + c * (Rpad / 32) + (out_r / 32) + b);
            }
        }
        out_r += len;
    }
}

ORACLE_API void oracle_mxfp8_quantize(const float *x, int64_t rows, int64_t cols, int axis,
                                      const int32_t *seg_off, int32_t nseg, uint64_t seed,
                                      uint64_t offset, int rounding, uint8_t *codes,
                                      uint8_t *scales) {
    oracle_mxfp8_quantize_at(x, rows, cols, 0, axis, seg_off, nseg, seed, offset, rounding, codes,
                             scales);
}

/* x_hat = e4m3(q) * 2^(e - 127), exact. layout as produced above with
 * n_rows x n_cols codes and n_cols/32 scales per row. */
ORACLE_API void oracle_mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales,
                                        int64_t n_rows, int64_t n_cols, float *out) {
    for (int64_t r = 0; r < n_rows; ++r)
        for (int64_t c = 0; c < n_cols; ++c)
            out[r * n_cols + c] = (float)(oracle_e4m3_decode(codes[r * n_cols + c]) *
                                          oracle_e8m0_decode(scales[r * (n_cols / 32) + c / 32]));
}

/* ------------------------------------------------------------------------ */
/* 32-point random Hadamard transform ([P2] "Key Takeaways" and              */
/* "Architecture highlights": a 32-dimensional random Hadamard transform     */
/* before the combine traffic is quantized into a block-scaled format).      */
/* ------------------------------------------------------------------------ */
/*
 * READING: v = c * H32 * (s .* x) per 32-block, H32 the Sylvester Hadamard
 * matrix, c = fp32(1/sqrt(32)) (orthonormal), s one vector of 32 random signs
 * shared by every block: s_i = -1 iff bit i of word 0 of
 * Philox4x32-10(key = sign_seed, counter = 0) is set. Evaluation order in
 * fp32: sign flip, then the five butterfly stages h = 1, 2, 4, 8, 16 with
 * (a, b) -> (a + b, a - b) on the index pairs (j, j + h), then the product
 * with c. The inverse applies the same butterflies to v, multiplies by c and
 * flips the signs.
 */
ORACLE_API uint32_t oracle_rht_signs(uint64_t sign_seed) {
    uint32_t ctr[4] = {0, 0, 0, 0};
    uint32_t key[2] = {(uint32_t)sign_seed, (uint32_t)(sign_seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[0];
}

static void fwht32_f32(float *t) {
    for (int h = 1; h < 32; h <<= 1)
        for (int j = 0; j < 32; ++j)
            if ((j & h) == 0) {
                float a = t[j], b = t[j + h];
                t[j] = a + b;
                t[j + h] = a - b;
            }
}

static float rht_c(void) { return (float)(1.0 / sqrt(32.0)); }

ORACLE_API void oracle_rht32_forward_f32(const float *x, uint32_t signs, float *v) {
    float t[32];
    for (int i = 0; i < 32; ++i) t[i] = ((signs >> i) & 1) ? -x[i] : x[i];
    fwht32_f32(t);
    float c = rht_c();
    for (int i = 0; i < 32; ++i) v[i] = t[i] * c;
}

ORACLE_API void oracle_rht32_inverse_f32(const float *v, uint32_t signs, float *x) {
    float t[32];
    for (int i = 0; i < 32; ++i) t[i] = v[i];
    fwht32_f32(t);
    float c = rht_c();
    for (int i = 0; i < 32; ++i) {
        float u = t[i] * c;
        x[i] = ((signs >> i) & 1) ? -u : u;
    }
}

/* Exact-arithmetic version (fp64, c = 1/sqrt(32) in fp64) for the pins. */
ORACLE_API void oracle_rht32_f64(const double *x, uint32_t signs, int inverse, double *y) {
    double t[32];
    for (int i = 0; i < 32; ++i) t[i] = (!inverse && ((signs >> i) & 1)) ? -x[i] : x[i];
    for (int h = 1; h < 32; h <<= 1)
        for (int j = 0; j < 32; ++j)
            if ((j & h) == 0) {
                double a = t[j], b = t[j + h];
                t[j] = a + b;
                t[j + h] = a - b;
            }
    double c = 1.0 / sqrt(32.0);
    for (int i = 0; i < 32; ++i) {
        double u = t[i] * c;
        y[i] = (inverse && ((signs >> i) & 1)) ? -u : u;
    }
}

/* max |v| over the RHT32 transform v of rows x cols values: the tensor amax an
 * NVFP4 payload takes, computed a slice of rows at a time for large tensors. */
ORACLE_API float oracle_rht32_amax(const float *x, int64_t rows, int64_t cols, uint64_t sign_seed) {
    uint32_t s = oracle_rht_signs(sign_seed);
    float v[32], amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 32; ++b) {
            oracle_rht32_forward_f32(x + r * cols + b * 32, s, v);
            for (int i = 0; i < 32; ++i)
                if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
        }
    return amax;
}

/*
 * RHT32 + block-scaled quantization of rows x cols values (cols % 32 == 0).
 * fmt 0 = NVFP4: the tensor amax is taken over the transformed values v (or
 *   given in amax_in) and each 32-block carries two 16-element NVFP4 blocks.
 *   codes [rows x cols/2], scales [rows x cols/16], *ts_out.
 * fmt 1 = MXFP8 (round-to-nearest-even): codes [rows x cols], scales
 *   [rows x cols/32]; ts_out untouched.
 */
ORACLE_API void oracle_rht32_quantize(const float *x, int64_t rows, int64_t cols,
                                      uint64_t sign_seed, int fmt, const float *amax_in,
                                      uint8_t *codes, uint8_t *scales, float *ts_out) {
    uint32_t s = oracle_rht_signs(sign_seed);
    float *v = (float *)malloc(sizeof(float) * (size_t)(rows * cols));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 32; ++b)
            oracle_rht32_forward_f32(x + r * cols + b * 32, s, v + r * cols + b * 32);
    if (fmt == 0) {
        oracle_nvfp4_quantize(v, rows, cols, amax_in, codes, scales, ts_out);
    } else {
        oracle_mxfp8_quantize(v, rows, cols, 0, NULL, 0, 0, 0, 0, codes, scales);
    }
    free(v);
}

ORACLE_API void oracle_rht32_dequantize(const uint8_t *codes, const uint8_t *scales, float ts,
                                        int64_t rows, int64_t cols, uint64_t sign_seed,
                                        int fmt, float *out) {
    uint32_t s = oracle_rht_signs(sign_seed);
    float *v = (float *)malloc(sizeof(float) * (size_t)(rows * cols));
    if (fmt == 0)
        oracle_nvfp4_dequantize(codes, scales, ts, rows, cols, v);
    else
        oracle_mxfp8_dequantize(codes, scales, rows, cols, v);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 32; ++b)
            oracle_rht32_inverse_f32(v + r * cols + b * 32, s, out + r * cols + b * 32);
    free(v);
}

/*
 * Combine straight from the RHT32-quantized payload (aicoder.com 'Key
 * Takeaways': the combine traffic travels block-scaled after a 32-point random
 * Hadamard transform).
 * READING: the transform is linear, so the weighted sum of a token's k rows is
 * taken in the transformed domain and one inverse transform per token
 * follows: sum_j w_j H^-1 v_j = H^-1 sum_j w_j v_j. Values are the exact
 * dequantized payload (NVFP4: e2m1 * e4m3 scale * ts; MXFP8: e4m3 * 2^k),
 * summed and transformed in fp64 (c = 1/sqrt(32) in fp64), rounded once to
 * bf16 (oracle_combine_rht) or returned in fp64 (oracle_combine_rht_f64).
 * codes/scales: rows x d payload in the ROWMAJOR layout of oracle_rht32_quantize.
 */
static double payload_value(const uint8_t *codes, const uint8_t *scales, float ts, int fmt,
                            int64_t d, int64_t r, int64_t c) {
    if (fmt == 0) {
        uint8_t byte = codes[r * (d / 2) + c / 2];
        uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
        return oracle_e2m1_decode(nib) * oracle_e4m3_decode(scales[r * (d / 16) + c / 16]) * (double)ts;
    }
    return oracle_e4m3_decode(codes[r * d + c]) * oracle_e8m0_decode(scales[r * (d / 32) + c / 32]);
}

ORACLE_API void oracle_combine_rht_f64(const uint8_t *codes, const uint8_t *scales, float ts,
                                       int fmt, uint64_t sign_seed, const int32_t *pos,
                                       const double *w, int64_t T, int32_t k, int64_t d,
                                       double *out) {
    uint32_t s = oracle_rht_signs(sign_seed);
    for (int64_t t = 0; t < T; ++t)
        for (int64_t b = 0; b < d / 32; ++b) {
            double acc[32];
            for (int i = 0; i < 32; ++i) {
                double sum = 0.0;
                for (int j = 0; j < k; ++j)
                    sum += w[t * k + j] * payload_value(codes, scales, ts, fmt, d, pos[t * k + j], b * 32 + i);
                acc[i] = sum;
            }
            oracle_rht32_f64(acc, s, 1, out + t * d + b * 32);
        }
}

ORACLE_API void oracle_combine_rht(const uint8_t *codes, const uint8_t *scales, float ts, int fmt,
                                   uint64_t sign_seed, const int32_t *pos, const double *w,
                                   int64_t T, int32_t k, int64_t d, uint16_t *out_bits) {
    double *x = (double *)malloc(sizeof(double) * (size_t)(T * d));
    oracle_combine_rht_f64(codes, scales, ts, fmt, sign_seed, pos, w, T, k, d, x);
    for (int64_t i = 0; i < T * d; ++i) out_bits[i] = oracle_bf16_from_f64(x[i]);
    free(x);
}

/* ------------------------------------------------------------------------ */
/* Routing and permutation ([P4] "PART 01": 384 experts, 8 routed per token) */
/* ------------------------------------------------------------------------ */
/*
 * READING: probabilities are the softmax of the router logits; the k experts
 * with the largest logits are chosen (largest first, a tie goes to the lower
 * expert id), which is the same set as the largest probabilities; the weight
 * of slot j is p_j / sum of the k chosen p (renorm = 1) or p_j (renorm = 0).
 * No capacity limit, no dropped tokens.
 */
ORACLE_API void oracle_route(const float *logits, int64_t T, int32_t E, int32_t k, int renorm,
                             int32_t *topk_idx, double *topk_w) {
    char *taken = (char *)malloc((size_t)E);
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        double mx = -INFINITY;
        for (int e = 0; e < E; ++e) if ((double)l[e] > mx) mx = l[e];
        double z = 0.0;
        for (int e = 0; e < E; ++e) { p[e] = exp((double)l[e] - mx); z += p[e]; }
        for (int e = 0; e < E; ++e) p[e] /= z;
        memset(taken, 0, (size_t)E);
        double sel = 0.0;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
            taken[best] = 1;
            topk_idx[t * k + j] = best;
            topk_w[t * k + j] = p[best];
            sel += p[best];
        }
        if (renorm)
            for (int j = 0; j < k; ++j) topk_w[t * k + j] /= sel;
    }
    free(taken);
    free(p);
}

/*
 * READING: routed slots (t, j) are grouped by expert with a counting sort that
 * keeps ascending (t, j) order inside each expert; each expert's block of rows
 * starts at a multiple of 128 (expert_off[e], expert_off[E] = total padded
 * rows); pos[t*k + j] is the row of slot (t, j); token_of[row] is its token or
 * -1 for a padding row. token_of must hold rp_max entries.
 */
ORACLE_API void oracle_permute(const int32_t *topk_idx, int64_t T, int32_t E, int32_t k,
                               int64_t rp_max, int32_t *expert_off, int32_t *pos,
                               int32_t *token_of) {
    int64_t *cnt = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int64_t i = 0; i < T * k; ++i) cnt[topk_idx[i]]++;
    int64_t acc = 0;
    for (int e = 0; e < E; ++e) {
        expert_off[e] = (int32_t)acc;
        acc += (cnt[e] + 127) / 128 * 128;
    }
    expert_off[E] = (int32_t)acc;
    for (int64_t r = 0; r < rp_max; ++r) token_of[r] = -1;
    int64_t *fill = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = topk_idx[t * k + j];
            int64_t row = expert_off[e] + fill[e]++;
            pos[t * k + j] = (int32_t)row;
            token_of[row] = (int32_t)t;
        }
    free(cnt);
    free(fill);
}

/* ------------------------------------------------------------------------ */
/* GEMM and the expert FFN                                                   */
/* ------------------------------------------------------------------------ */

/* C[m][n] = sum_k A[m][k] * B[n][k] in fp64, k ascending. Rows are independent,
 * so they may run in parallel without changing any result. */
ORACLE_API void oracle_gemm_f64(const double *A, const double *B, int64_t M, int64_t N,
                                int64_t K, double *C) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const double *a = A + m * K, *b = B + n * K;
            double s = 0.0;
            for (int64_t kk = 0; kk < K; ++kk) s += a[kk] * b[kk];
            C[m * N + n] = s;
        }
}

/* Dequantize an NVFP4 matrix (row-major scales) to fp64, including ts. */
ORACLE_API void oracle_nvfp4_to_f64(const uint8_t *codes, const uint8_t *scales, float ts,
                                    int64_t rows, int64_t cols, double *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = nvfp4_value(codes, scales, ts, cols, r, c);
}

/* READING: SwiGLU h = silu(g) * u with silu(g) = g / (1 + exp(-g)); the first
 * f rows of W1 give g, the next f rows give u. */
static double swiglu(double g, double u) { return g / (1.0 + exp(-g)) * u; }

ORACLE_API double oracle_swiglu(double g, double u) { return swiglu(g, u); }

/*
 * One expert of the FFN forward, in the order the layer computes it:
 *   gu = dq(xq) * dq(W1_e)^T                (fp64, dq includes the tensor scales)
 *   h  = bf16(silu(g) * u)
 *   h_amax = max|h| over the expert's rows; hq = NVFP4(h) with that amax
 *   y  = bf16(dq(hq) * dq(W2_e)^T)
 * xq: n rows (codes d/2 bytes, scales d/16), W1: 2f x d, W2: d x f.
 * Outputs h_bits [n x f], hq [n x f/2], hq_sc [n x f/16], *h_ts, y_bits [n x d].
 * Rows listed in rows_out (count n_out, indices into 0..n-1) are the only y
 * rows written (all rows when rows_out is NULL); h is always computed for
 * every row because the expert's amax needs it.
 */
ORACLE_API void oracle_expert_ffn(const uint8_t *xq, const uint8_t *xq_sc, float x_ts, int64_t n,
                                  int64_t d, int64_t f, const uint8_t *w1, const uint8_t *w1_sc,
                                  float w1_ts, const uint8_t *w2, const uint8_t *w2_sc,
                                  float w2_ts, const int32_t *rows_out, int64_t n_out,
                                  uint16_t *h_bits, uint8_t *hq, uint8_t *hq_sc, float *h_ts,
                                  uint16_t *y_bits) {
    double *A = (double *)malloc(sizeof(double) * (size_t)(n * d));
    double *B1 = (double *)malloc(sizeof(double) * (size_t)(2 * f * d));
    double *GU = (double *)malloc(sizeof(double) * (size_t)(n * 2 * f));
    oracle_nvfp4_to_f64(xq, xq_sc, x_ts, n, d, A);
    oracle_nvfp4_to_f64(w1, w1_sc, w1_ts, 2 * f, d, B1);
    oracle_gemm_f64(A, B1, n, 2 * f, d, GU);
    free(B1);
    float *hf = (float *)malloc(sizeof(float) * (size_t)(n * f));
    for (int64_t r = 0; r < n; ++r)
        for (int64_t c = 0; c < f; ++c) {
            uint16_t hb = oracle_bf16_from_f64(swiglu(GU[r * 2 * f + c], GU[r * 2 * f + f + c]));
            h_bits[r * f + c] = hb;
            hf[r * f + c] = oracle_bf16_to_f32(hb);
        }
    free(GU);
    oracle_nvfp4_quantize(hf, n, f, NULL, hq, hq_sc, h_ts);
    free(hf);
    double *H = (double *)malloc(sizeof(double) * (size_t)(n * f));
    double *B2 = (double *)malloc(sizeof(double) * (size_t)(d * f));
    oracle_nvfp4_to_f64(hq, hq_sc, *h_ts, n, f, H);
    oracle_nvfp4_to_f64(w2, w2_sc, w2_ts, d, f, B2);
    int64_t cnt = rows_out ? n_out : n;
    double *Hs = (double *)malloc(sizeof(double) * (size_t)(cnt * f));
    for (int64_t i = 0; i < cnt; ++i)
        memcpy(Hs + i * f, H + (rows_out ? rows_out[i] : i) * f, sizeof(double) * (size_t)f);
    double *Y = (double *)malloc(sizeof(double) * (size_t)(cnt * d));
    oracle_gemm_f64(Hs, B2, cnt, d, f, Y);
    for (int64_t i = 0; i < cnt * d; ++i) y_bits[i] = oracle_bf16_from_f64(Y[i]);
    free(A); free(H); free(B2); free(Hs); free(Y);
}

/* Dequantize an MXFP8 matrix (row-major E8M0 scales, blocks of 32 along
 * columns) to fp64. */
static void mxfp8_to_f64(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                         double *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = oracle_e4m3_decode(codes[r * cols + c]) *
                                ldexp(1.0, (int)scales[r * (cols / 32) + c / 32] - 127);
}

/*
 * READING ([P2] "Architecture highlights": the last 16.6% of layers stay in
 * MXFP8): the same expert forward as oracle_expert_ffn with every operand in
 * MXFP8 instead of NVFP4: E4M3 codes with one E8M0 scale per 32 consecutive
 * elements of a row, rounded to nearest-even (stochastic rounding is for the
 * gradients), no tensor scale.
 *   gu = dq(xq) * dq(W1_e)^T                (fp64)
 *   h  = bf16(silu(g) * u)
 *   hq = MXFP8(h) along rows, round-to-nearest-even
 *   y  = bf16(dq(hq) * dq(W2_e)^T)
 * xq: n x d codes + n x d/32 scales, W1: 2f x d, W2: d x f (row-major scales).
 * Outputs h_bits [n x f], hq [n x f], hq_sc [n x f/32], y_bits [n_out or n
 * rows x d]; rows_out as in oracle_expert_ffn.
 */
ORACLE_API void oracle_expert_ffn_mxfp8(const uint8_t *xq, const uint8_t *xq_sc, int64_t n,
                                        int64_t d, int64_t f, const uint8_t *w1,
                                        const uint8_t *w1_sc, const uint8_t *w2,
                                        const uint8_t *w2_sc, const int32_t *rows_out,
                                        int64_t n_out, uint16_t *h_bits, uint8_t *hq,
                                        uint8_t *hq_sc, uint16_t *y_bits) {
    double *A = (double *)malloc(sizeof(double) * (size_t)(n * d));
    double *B1 = (double *)malloc(sizeof(double) * (size_t)(2 * f * d));
    double *GU = (double *)malloc(sizeof(double) * (size_t)(n * 2 * f));
    mxfp8_to_f64(xq, xq_sc, n, d, A);
    mxfp8_to_f64(w1, w1_sc, 2 * f, d, B1);
    oracle_gemm_f64(A, B1, n, 2 * f, d, GU);
    free(A);
    free(B1);
    float *hf = (float *)malloc(sizeof(float) * (size_t)(n * f));
    for (int64_t r = 0; r < n; ++r)
        for (int64_t c = 0; c < f; ++c) {
            uint16_t hb = oracle_bf16_from_f64(swiglu(GU[r * 2 * f + c], GU[r * 2 * f + f + c]));
            h_bits[r * f + c] = hb;
            hf[r * f + c] = oracle_bf16_to_f32(hb);
        }
    free(GU);
    oracle_mxfp8_quantize(hf, n, f, 0, NULL, 0, 0, 0, 0, hq, hq_sc);
    free(hf);
    double *H = (double *)malloc(sizeof(double) * (size_t)(n * f));
    double *B2 = (double *)malloc(sizeof(double) * (size_t)(d * f));
    mxfp8_to_f64(hq, hq_sc, n, f, H);
    mxfp8_to_f64(w2, w2_sc, d, f, B2);
    int64_t cnt = rows_out ? n_out : n;
    double *Hs = (double *)malloc(sizeof(double) * (size_t)(cnt * f));
    for (int64_t i = 0; i < cnt; ++i)
        memcpy(Hs + i * f, H + (rows_out ? rows_out[i] : i) * f, sizeof(double) * (size_t)f);
    double *Y = (double *)malloc(sizeof(double) * (size_t)(cnt * d));
    oracle_gemm_f64(Hs, B2, cnt, d, f, Y);
    for (int64_t i = 0; i < cnt * d; ++i) y_bits[i] = oracle_bf16_from_f64(Y[i]);
    free(H); free(B2); free(Hs); free(Y);
}

/*
 * READING ([P1] "训练数值格式分工清单": the backward pass of the expert layers
 * runs in MXFP8): the SwiGLU step of the backward pass. For h = silu(g) * u
 * with silu(g) = g * s(g), s(g) = 1 / (1 + exp(-g)):
 *   dg = dh * u * s(g) * (1 + g * (1 - s(g)))
 *   du = dh * silu(g)
 * gu_bits [rows x 2f] holds g in columns 0..f-1 and u in f..2f-1 (the layout
 * GEMM1 writes), dh_bits [rows x f]; dgu_bits [rows x 2f] gets dg | du in the
 * same layout, each computed in fp64 and rounded once to bf16.
 */
ORACLE_API void oracle_swiglu_bwd(const uint16_t *gu_bits, const uint16_t *dh_bits, int64_t rows,
                                  int64_t f, uint16_t *dgu_bits) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < f; ++c) {
            const double g = oracle_bf16_to_f32(gu_bits[r * 2 * f + c]);
            const double u = oracle_bf16_to_f32(gu_bits[r * 2 * f + f + c]);
            const double dh = oracle_bf16_to_f32(dh_bits[r * f + c]);
            const double sg = 1.0 / (1.0 + exp(-g));
            dgu_bits[r * 2 * f + c] = oracle_bf16_from_f64(dh * u * sg * (1.0 + g * (1.0 - sg)));
            dgu_bits[r * 2 * f + f + c] = oracle_bf16_from_f64(dh * g * sg);
        }
}

/*
 * READING ([P2] "Key Takeaways": the combine step): out[t] = sum over slots j
 * of w[t, j] * y[pos[t, j]] in fp64, rounded once to bf16. y rows are bf16.
 */
ORACLE_API void oracle_combine(const uint16_t *y_bits, const int32_t *pos, const double *w,
                               int64_t T, int32_t k, int64_t d, uint16_t *out_bits) {
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < d; ++c) {
            double s = 0.0;
            for (int j = 0; j < k; ++j)
                s += w[t * k + j] * (double)oracle_bf16_to_f32(y_bits[(int64_t)pos[t * k + j] * d + c]);
            out_bits[t * d + c] = oracle_bf16_from_f64(s);
        }
}

/* Same, for a payload given as fp32 rows (a dequantized combine payload). */
ORACLE_API void oracle_combine_f32(const float *y, const int32_t *pos, const double *w, int64_t T,
                                   int32_t k, int64_t d, uint16_t *out_bits) {
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < d; ++c) {
            double s = 0.0;
            for (int j = 0; j < k; ++j)
                s += w[t * k + j] * (double)y[(int64_t)pos[t * k + j] * d + c];
            out_bits[t * d + c] = oracle_bf16_from_f64(s);
        }
}
