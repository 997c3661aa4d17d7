/*
 * qmv_oracle.c -- plain, slow fp64 CPU oracle for the weight-quantized
 * matrix-vector product  y[m,n] = sum_k x[m,k] * dequant(W)[n,k].
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: it is used by tests/, by __graft_entry__.smoke() and by the
 * cpu_baseline / reference leg of bench.py, nowhere else.  It shares no code,
 * header, table or constant with the CUDA library: every decoder below is
 * written from the format definitions on the pages it cites.
 *
 * Sources (page title, section):
 *  - MLX "quantized_nax.h" (mlx 1.0.0 source page), functions get_pack_factor,
 *    get_bytes_per_pack, qdot, dequantize: affine pack geometry, LSB-first
 *    code order inside a pack, and w = scale * q + bias.
 *  - "wh-iron kernel-op coverage audit", section "Quantization precision
 *    coverage", Track 1 table and the E2M1 / E4M3 / E8M0 codec notes:
 *    MXFP4 = E2M1 x E8M0 per 32, NVFP4 = E2M1 x E4M3 per 16 x FP32 global,
 *    MXFP8 = E4M3 x E8M0 per 32; E4M3 has 3 mantissa bits, exponent bias 7,
 *    max 448 and an explicit NaN code; the rest of the Track 1 table (E5M2,
 *    NVFP8, the FP32-scale legacy formats, the symmetric int / mxint
 *    family and the FP16-scale twins) in oracle_qmv_block_scaled.
 *  - MLX pull request "affine_qmv_fast_rows / fp_qmv_fast_rows", description:
 *    the sum(x) bias term is formed from values widened before accumulation.
 *    The oracle has no such issue: it evaluates every product and sum in fp64.
 *
 * Every function is a direct statement of a definition; there is no blocking,
 * fusion or reordering.  Parity status of each function is listed in the
 * tests that pin it (tests/test_oracle_pins.py); every exported function here
 * is pinned there, none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stddef.h>

/* dtype codes used on the oracle's own ctypes boundary */
enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2 };
/* FP weight modes */
enum { OR_MXFP4 = 0, OR_NVFP4 = 1, OR_MXFP8 = 2 };

/* ---------------------------------------------------------------------------
 * Element types of x, y, scales and biases, widened exactly to fp64.
 * binary16 and bfloat16 are decoded from their IEEE-style field definitions.
 * ------------------------------------------------------------------------- */
double oracle_f16_value(uint32_t h) {
    uint32_t s = (h >> 15) & 1u, e = (h >> 10) & 31u, m = h & 1023u;
    double v;
    if (e == 0) v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31) v = (m == 0) ? INFINITY : NAN;
    else v = ldexp(1.0 + (double)m / 1024.0, (int)e - 15);
    return s ? -v : v;
}

double oracle_bf16_value(uint32_t h) {
    uint32_t s = (h >> 15) & 1u, e = (h >> 7) & 255u, m = h & 127u;
    double v;
    if (e == 0) v = ldexp((double)m, -133);                /* subnormal: m * 2^-133 */
    else if (e == 255) v = (m == 0) ? INFINITY : NAN;
    else v = ldexp(1.0 + (double)m / 128.0, (int)e - 127);
    return s ? -v : v;
}

static double load_elem(const void* p, size_t i, int dtype) {
    if (dtype == OR_F32) { float f; memcpy(&f, (const char*)p + 4 * i, 4); return (double)f; }
    uint16_t h; memcpy(&h, (const char*)p + 2 * i, 2);
    return dtype == OR_F16 ? oracle_f16_value(h) : oracle_bf16_value(h);
}

/* ---------------------------------------------------------------------------
 * Affine pack geometry (MLX quantized_nax.h, get_pack_factor /
 * get_bytes_per_pack with an 8-bit word): 3- and 5-bit codes come 8 to a pack
 * of 3 or 5 bytes, 6-bit codes 4 to a pack of 3 bytes, and 2/4/8-bit codes
 * 8/bits to a single byte.
 * ------------------------------------------------------------------------- */
int oracle_pack_factor(int bits) {
    if (bits == 3 || bits == 5) return 8;
    if (bits == 6) return 4;
    return 8 / bits;
}

int oracle_bytes_per_pack(int bits) {
    if ((bits & (bits - 1)) == 0) return 1;
    return bits == 5 ? 5 : 3;
}

/* Row byte length K_w = K * bytes_per_pack / pack_factor (= K * bits / 8). */
long long oracle_row_bytes(long long K, int bits) {
    return K * oracle_bytes_per_pack(bits) / oracle_pack_factor(bits);
}

/* Code i of a packed row.  Inside a pack the codes are read least significant
 * bit first: with the pack's bytes taken as one little-endian integer, code j
 * of the pack occupies bits [bits*j, bits*j + bits).  This single reading is
 * what the masks of MLX's qdot / dequantize select for every width. */
uint32_t oracle_affine_code(const uint8_t* row, long long i, int bits) {
    int pf = oracle_pack_factor(bits), bpp = oracle_bytes_per_pack(bits);
    long long p = i / pf;
    int j = (int)(i % pf);
    uint64_t v = 0;
    for (int b = 0; b < bpp; ++b) v |= (uint64_t)row[p * bpp + b] << (8 * b);
    return (uint32_t)((v >> (bits * j)) & ((1u << bits) - 1u));
}

/* ---------------------------------------------------------------------------
 * Micro-float codecs (wh-iron audit, Track 1 and the codec notes).
 * ------------------------------------------------------------------------- */
/* E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN. */
double oracle_e2m1(uint32_t c) {
    uint32_t s = (c >> 3) & 1u, e = (c >> 1) & 3u, m = c & 1u;
    double v = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -v : v;
}

/* E4M3 (OCP "FN" flavour): sign, 4 exponent bits (bias 7), 3 mantissa bits;
 * exponent field 0 is subnormal; S.1111.111 is NaN; no infinities. */
double oracle_e4m3(uint32_t c) {
    uint32_t s = (c >> 7) & 1u, e = (c >> 3) & 15u, m = c & 7u;
    double v;
    if ((c & 0x7Fu) == 0x7Fu) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -v : v;
}

/* E8M0: an unsigned power-of-two exponent byte, 2^(e - 127); 0xFF is NaN. */
double oracle_e8m0(uint32_t e) {
    if ((e & 0xFFu) == 0xFFu) return NAN;
    return ldexp(1.0, (int)(e & 0xFFu) - 127);
}

/* ---------------------------------------------------------------------------
 * One correctly rounded fp32 value of the exact sum a + b (a, b exact fp64).
 * The fp64 sum is first rounded to odd (TwoSum gives its exact error), which
 * makes the following fp64 -> fp32 conversion a single correct rounding
 * (53 >= 24 + 2 bits).  Used for the dequantized fp32 weight
 * round_f32(scale * q + bias).
 * ------------------------------------------------------------------------- */
float oracle_round_f32_sum(double a, double b) {
    double s = a + b;
    double bb = s - a;
    double err = (a - (s - bb)) + (b - bb);            /* exact: a + b = s + err */
    if (err != 0.0 && isfinite(s)) {
        uint64_t u; memcpy(&u, &s, 8);
        if ((u & 1u) == 0) {                               /* even: step toward err */
            s = nextafter(s, err > 0 ? INFINITY : -INFINITY);
        }
    }
    return (float)s;
}

/* Exact dequantized affine weight (fp64) of element (n, k). */
static double affine_w(const uint8_t* w, const void* scales, const void* biases,
                       long long n, long long k, long long K, int bits, int group, int dtype) {
    const uint8_t* row = w + n * oracle_row_bytes(K, bits);
    long long gi = n * (K / group) + k / group;
    double s = load_elem(scales, (size_t)gi, dtype);
    double b = load_elem(biases, (size_t)gi, dtype);
    return s * (double)oracle_affine_code(row, k, bits) + b;
}

/* fp32 dequantized affine weights, out[n*K + k] = round_f32(scale*q + bias),
 * rows [n0, n1). */
void oracle_dequant_affine_f32(const uint8_t* w, const void* scales, const void* biases,
                               float* out, long long N, long long K, int bits, int group,
                               int dtype, long long n0, long long n1) {
    (void)N;
    for (long long n = n0; n < n1; ++n) {
        const uint8_t* row = w + n * oracle_row_bytes(K, bits);
        for (long long k = 0; k < K; ++k) {
            long long gi = n * (K / group) + k / group;
            double s = load_elem(scales, (size_t)gi, dtype);
            double b = load_elem(biases, (size_t)gi, dtype);
            double sq = s * (double)oracle_affine_code(row, k, bits); /* exact: <= 32 bits */
            out[n * K + k] = oracle_round_f32_sum(sq, b);
        }
    }
}

/* Dequantized affine weights in fp64: w = scale * q + bias with the stored
 * scale and bias widened exactly (MLX quantized_nax.h, dequantize).  The
 * product is exact (at most 32 significant bits); the sum is exact whenever
 * it fits 53 bits, which every f16 / bf16 scale and bias does (an f32 pair
 * could exceed that only with exponents more than 29 apart, where the one
 * fp64 rounding is far below any tolerance here).  Rows [n0, n1) of out
 * [N, K]. */
void oracle_dequant_affine_f64(const uint8_t* w, const void* scales, const void* biases,
                               double* out, long long N, long long K, int bits, int group,
                               int dtype, long long n0, long long n1) {
    (void)N;
    for (long long n = n0; n < n1; ++n) {
        const uint8_t* row = w + n * oracle_row_bytes(K, bits);
        for (long long k = 0; k < K; ++k) {
            long long gi = n * (K / group) + k / group;
            double s = load_elem(scales, (size_t)gi, dtype);
            double b = load_elem(biases, (size_t)gi, dtype);
            out[n * K + k] = s * (double)oracle_affine_code(row, k, bits) + b;
        }
    }
}

/* Block size along K and per-element width of each FP mode. */
static int fp_block(int mode) { return mode == OR_NVFP4 ? 16 : 32; }
static int fp_bits(int mode) { return mode == OR_MXFP8 ? 8 : 4; }

/* Exact dequantized FP weight (fp64) of element (n, k).  Codes are 4-bit
 * (two per byte, even k in the low nibble) or one byte each; one scale byte
 * per block; NVFP4 multiplies by the tensor-wide fp32 global scale. */
static double fp_w(const uint8_t* w, const uint8_t* scales, double global,
                   long long n, long long k, long long K, int mode) {
    int bits = fp_bits(mode), blk = fp_block(mode);
    const uint8_t* row = w + n * (K * bits / 8);
    uint32_t code = (bits == 8) ? row[k] : ((row[k / 2] >> (4 * (k % 2))) & 0xFu);
    uint32_t sc = scales[n * (K / blk) + k / blk];
    double e = (bits == 8) ? oracle_e4m3(code) : oracle_e2m1(code);
    if (mode == OR_NVFP4) return e * oracle_e4m3(sc) * global;
    return e * oracle_e8m0(sc);
}

/* fp32 dequantized FP weights; every product is exact in fp64 (at most 30
 * significant bits), so the cast is the one rounding. */
void oracle_dequant_fp_f32(const uint8_t* w, const uint8_t* scales, float global,
                           float* out, long long N, long long K, int mode,
                           long long n0, long long n1) {
    (void)N;
    for (long long n = n0; n < n1; ++n)
        for (long long k = 0; k < K; ++k)
            out[n * K + k] = (float)fp_w(w, scales, (double)global, n, k, K, mode);
}

/* ---------------------------------------------------------------------------
 * The product itself: y[m*N + n] = sum_k x[m,k] * w_hat[n,k] in fp64, plus
 * absdot[m*N + n] = sum_k |x[m,k] * w_hat[n,k]| (the size of the terms, used
 * by the tests' cancellation-aware tolerance).  Rows [n0, n1) only, so the
 * caller can sample rows or split them over threads.
 * ------------------------------------------------------------------------- */
void oracle_qmv_affine(const void* x, const uint8_t* w, const void* scales, const void* biases,
                       double* y, double* absdot, long long M, long long N, long long K,
                       int bits, int group, int dtype, long long n0, long long n1) {
    for (long long n = n0; n < n1; ++n)
        for (long long m = 0; m < M; ++m) {
            double acc = 0.0, aacc = 0.0;
            for (long long k = 0; k < K; ++k) {
                double t = load_elem(x, (size_t)(m * K + k), dtype) *
                           affine_w(w, scales, biases, n, k, K, bits, group, dtype);
                acc += t;
                aacc += fabs(t);
            }
            y[m * N + n] = acc;
            if (absdot) absdot[m * N + n] = aacc;
        }
}

/* ---------------------------------------------------------------------------
 * qvm: x times a weight matrix stored [K, N] (MLX quantized_nax.h, qouter,
 * the outer-product accumulate result[j] += x * (scale * q_j + bias); the
 * wh-iron audit's qvm family, "x.W with W [K, N]").  Row k of w packs the N
 * codes of the output columns LSB first exactly like a qmv row, with scales
 * and biases [K, N / group] grouped along N:
 *     y[m, n] = sum_k x[m, k] * (scale[k, n/group] * q[k, n] + bias[k, n/group])
 * Products and sum in fp64 as in oracle_qmv_affine.  Columns [n0, n1).
 * ------------------------------------------------------------------------- */
void oracle_qvm_affine(const void* x, const uint8_t* w, const void* scales, const void* biases,
                       double* y, double* absdot, long long M, long long N, long long K,
                       int bits, int group, int dtype, long long n0, long long n1) {
    for (long long n = n0; n < n1; ++n)
        for (long long m = 0; m < M; ++m) {
            double acc = 0.0, aacc = 0.0;
            for (long long k = 0; k < K; ++k) {
                /* element (k, n): row k, position n of a row of N codes */
                double t = load_elem(x, (size_t)(m * K + k), dtype) *
                           affine_w(w, scales, biases, k, n, N, bits, group, dtype);
                acc += t;
                aacc += fabs(t);
            }
            y[m * N + n] = acc;
            if (absdot) absdot[m * N + n] = aacc;
        }
}

void oracle_qmv_fp(const void* x, const uint8_t* w, const uint8_t* scales, float global,
                   double* y, double* absdot, long long M, long long N, long long K,
                   int mode, int dtype, long long n0, long long n1) {
    for (long long n = n0; n < n1; ++n)
        for (long long m = 0; m < M; ++m) {
            double acc = 0.0, aacc = 0.0;
            for (long long k = 0; k < K; ++k) {
                double t = load_elem(x, (size_t)(m * K + k), dtype) *
                           fp_w(w, scales, (double)global, n, k, K, mode);
                acc += t;
                aacc += fabs(t);
            }
            y[m * N + n] = acc;
            if (absdot) absdot[m * N + n] = aacc;
        }
}

/* ---------------------------------------------------------------------------
 * The Track-1 symmetric block-scaled formats (wh-iron kernel-op coverage
 * audit, "Quantization precision coverage": the three axes element / scale /
 * zero point, the Track 1 table, and the paragraph under it).  A weight
 * [N, K] is cut along K into contiguous blocks; every element is a code,
 * every block has one scale, there is no zero point, and the weight is
 *     w_hat[n, k] = element(code[n, k]) * scale[n, k / block]  (* global),
 * the tensor-wide FP32 global only for NVFP4.
 *   element: E2M1, E4M3, E5M2, or a signed integer of 2..8 bits (the
 *            audit's "signed integer ... float sign-extend": two's
 *            complement, range -2^(b-1) .. 2^(b-1) - 1);
 *   codes:   per row an LSB-first bit stream of b-bit codes, b the element
 *            width (the audit: "tight-bit-pack LSB-first into u32 words", a
 *            4-bit stream byte-identical to the nibble layout, 8-bit one byte
 *            per code), read with oracle_affine_code;
 *   scale:   E8M0 or E4M3 bytes, FP32 (4 B) or FP16 (2 B, the "*_f16"
 *            twins), stored [N, K / block] row-major.
 * ------------------------------------------------------------------------- */
enum { OR_EL_E2M1 = 0, OR_EL_E4M3 = 1, OR_EL_E5M2 = 2, OR_EL_INT = 3 };
enum { OR_SC_E8M0 = 0, OR_SC_E4M3 = 1, OR_SC_F32 = 2, OR_SC_F16 = 3 };

/* E5M2: sign, 5 exponent bits (bias 15), 2 mantissa bits, with IEEE
 * semantics: exponent field 0 is subnormal, 31 is infinity (mantissa 0) or
 * NaN.  The audit's KV-cache row gives its largest finite value, 57344. */
double oracle_e5m2(uint32_t c) {
    c &= 0xFFu;
    const double s = (c & 0x80u) ? -1.0 : 1.0;
    const int e = (int)((c >> 2) & 31u), m = (int)(c & 3u);
    if (e == 31) return m ? NAN : s * INFINITY;
    if (e == 0) return s * ((double)m / 4.0) * ldexp(1.0, -14);
    return s * (1.0 + (double)m / 4.0) * ldexp(1.0, e - 15);
}

/* Signed integer element of `bits` bits (2..8) from its raw field: two's
 * complement, so a field with the top bit set is field - 2^bits. */
double oracle_sint(uint32_t q, int bits) {
    q &= (1u << bits) - 1u;
    return (q >> (bits - 1)) ? (double)q - ldexp(1.0, bits) : (double)q;
}

/* Element k of a row. */
static double bs_elem(const uint8_t* row, long long k, int elem, int bits) {
    const uint32_t c = oracle_affine_code(row, k, bits);
    switch (elem) {
        case OR_EL_E2M1: return oracle_e2m1(c);
        case OR_EL_E4M3: return oracle_e4m3(c);
        case OR_EL_E5M2: return oracle_e5m2(c);
        default: return oracle_sint(c, bits);
    }
}

/* Block scale i of the scale array, widened exactly. */
double oracle_block_scale(const void* s, long long i, int kind) {
    switch (kind) {
        case OR_SC_E8M0: return oracle_e8m0(((const uint8_t*)s)[i]);
        case OR_SC_E4M3: return oracle_e4m3(((const uint8_t*)s)[i]);
        case OR_SC_F32: { float f; memcpy(&f, (const char*)s + 4 * i, 4); return (double)f; }
        default: { uint16_t h; memcpy(&h, (const char*)s + 2 * i, 2); return oracle_f16_value(h); }
    }
}

/* Exact dequantized weight (fp64) of element (n, k).  Every product is exact:
 * an element has at most 8 significant bits, an E8M0 / E4M3 / FP16 / FP32
 * scale at most 24, and the NVFP4 global (24) meets an E2M1 x E4M3 product
 * of at most 6. */
static double bs_w(const uint8_t* w, const void* scales, int use_global, double global, long long n,
                   long long k, long long K, int elem, int bits, int block, int kind) {
    const uint8_t* row = w + n * (K * bits / 8);
    const double v = bs_elem(row, k, elem, bits) * oracle_block_scale(scales, n * (K / block) + k / block, kind);
    return use_global ? v * global : v;
}

/* fp32 dequantized Track-1 weights (the exact value, one rounding). */
void oracle_dequant_block_scaled_f32(const uint8_t* w, const void* scales, int use_global, float global,
                                     float* out, long long N, long long K, int elem, int bits, int block,
                                     int kind, long long n0, long long n1) {
    (void)N;
    for (long long n = n0; n < n1; ++n)
        for (long long k = 0; k < K; ++k)
            out[n * K + k] = (float)bs_w(w, scales, use_global, (double)global, n, k, K, elem, bits, block, kind);
}

/* y[m, n] = sum_k x[m, k] * w_hat[n, k] in fp64 (and absdot), rows [n0, n1). */
void oracle_qmv_block_scaled(const void* x, const uint8_t* w, const void* scales, int use_global, float global,
                             double* y, double* absdot, long long M, long long N, long long K, int elem,
                             int bits, int block, int kind, int dtype, long long n0, long long n1) {
    for (long long n = n0; n < n1; ++n)
        for (long long m = 0; m < M; ++m) {
            double acc = 0.0, aacc = 0.0;
            for (long long k = 0; k < K; ++k) {
                double t = load_elem(x, (size_t)(m * K + k), dtype) *
                           bs_w(w, scales, use_global, (double)global, n, k, K, elem, bits, block, kind);
                acc += t;
                aacc += fabs(t);
            }
            y[m * N + n] = acc;
            if (absdot) absdot[m * N + n] = aacc;
        }
}

/* ---------------------------------------------------------------------------
 * Rounding fp32 to the element types, to nearest, ties to even (IEEE 754
 * roundTiesToEven), from the field definitions above.  Finite inputs.
 * ------------------------------------------------------------------------- */
/* bfloat16 keeps fp32's sign and exponent and the top 7 mantissa bits: the
 * dropped low 16 bits decide the rounding (above half up, below down, exactly
 * half to the even neighbour). */
uint32_t oracle_f32_to_bf16(float f) {
    uint32_t u; memcpy(&u, &f, 4);
    uint32_t lo = u & 0xFFFFu, hi = u >> 16;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;   /* a carry into the exponent is correct */
    return hi & 0xFFFFu;
}

/* binary16: |v| >= 65520 rounds to infinity; below 2^-14 the value is an
 * integer multiple of 2^-24 (subnormal); otherwise 1.m * 2^e with 10 mantissa
 * bits.  Scaling by powers of two is exact in fp64, and nearbyint rounds ties
 * to even under the default rounding mode. */
uint32_t oracle_f32_to_f16(float f) {
    double v = (double)f;
    uint32_t s = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a >= 65520.0) return s | 0x7C00u;
    if (a < ldexp(1.0, -14)) {
        double m = nearbyint(a * ldexp(1.0, 24));          /* 0..1024; 1024 encodes 2^-14 */
        return s | (uint32_t)m;
    }
    int e;
    double fr = frexp(a, &e);                              /* a = fr * 2^e, fr in [0.5, 1) */
    e -= 1;                                                /* a = (2 fr) * 2^e, 2 fr in [1, 2) */
    double m = nearbyint((2.0 * fr - 1.0) * 1024.0);
    if (m == 1024.0) { m = 0.0; e += 1; }
    return s | ((uint32_t)(e + 15) << 10) | (uint32_t)m;
}

/* ---------------------------------------------------------------------------
 * Affine quantizer (wh-iron kernel-op coverage audit, the "quantized
 * (affine_quantize / affine_dequantize)" row: quantize and dequantize for
 * every width; the audit's Track 2 describes the scheme as a min/max range
 * mapped to a scale and a bias).  The pages name these kernels but do not
 * state their arithmetic; this is the plainest reading consistent with the
 * dequantization w = scale*q + bias (MLX quantized_nax.h, dequantize), whose
 * inverse is the quotient (w - bias) / scale: for each group of `group`
 * consecutive weights of a row,
 *     bias  = min(w),  scale = (max(w) - min(w)) / (2^bits - 1),
 * both rounded to the element type, and
 *     q = nearest integer, ties to even, to (w - bias_T) / scale_T,
 * the difference and the quotient each one fp32 IEEE operation (one correctly
 * rounded division per weight), clamped to [0, 2^bits - 1].  q = 0 when
 * scale_T is 0 and when the quotient is NaN (an infinite difference over an
 * infinite scale, from a range beyond the fp32 maximum).  min and max are
 * taken in element order with strict comparisons, so of +0 and -0 the first
 * one met is kept.  Weights are finite.  Codes are packed LSB first exactly as
 * oracle_affine_code reads them.  Rows [n0, n1).
 * ------------------------------------------------------------------------- */
static float load_f32(const void* p, size_t i, int dtype) {
    return (float)load_elem(p, i, dtype);                  /* exact: every T is an fp32 value */
}

static float store_round(void* p, size_t i, int dtype, float v) {
    if (dtype == OR_F32) { memcpy((char*)p + 4 * i, &v, 4); return v; }
    uint16_t h = (uint16_t)(dtype == OR_F16 ? oracle_f32_to_f16(v) : oracle_f32_to_bf16(v));
    memcpy((char*)p + 2 * i, &h, 2);
    return (float)(dtype == OR_F16 ? oracle_f16_value(h) : oracle_bf16_value(h));
}

static void put_code(uint8_t* row, long long i, int bits, uint32_t code) {
    int pf = oracle_pack_factor(bits), bpp = oracle_bytes_per_pack(bits);
    long long p = i / pf;
    int j = (int)(i % pf);
    uint64_t v = (uint64_t)code << (bits * j);
    for (int b = 0; b < bpp; ++b) row[p * bpp + b] |= (uint8_t)(v >> (8 * b));
}

void oracle_quantize_affine(const void* w, uint8_t* wq, void* scales, void* biases, long long N,
                            long long K, int bits, int group, int dtype, long long n0, long long n1) {
    (void)N;
    const int qmax = (1 << bits) - 1;
    const long long rb = oracle_row_bytes(K, bits);
    for (long long n = n0; n < n1; ++n) {
        uint8_t* row = wq + n * rb;
        memset(row, 0, (size_t)rb);
        for (long long g0 = 0; g0 < K; g0 += group) {
            float lo = load_f32(w, (size_t)(n * K + g0), dtype), hi = lo;
            for (long long k = g0 + 1; k < g0 + group; ++k) {
                float v = load_f32(w, (size_t)(n * K + k), dtype);
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            const float range = hi - lo;                    /* fp32 */
            const float scale = range / (float)qmax;        /* fp32 */
            const size_t gi = (size_t)(n * (K / group) + g0 / group);
            const float sT = store_round(scales, gi, dtype, scale);
            const float bT = store_round(biases, gi, dtype, lo);
            for (long long k = g0; k < g0 + group; ++k) {
                uint32_t q = 0;
                if (sT != 0.0f) {
                    const float diff = load_f32(w, (size_t)(n * K + k), dtype) - bT;   /* fp32 */
                    const float d = diff / sT;                                          /* fp32 */
                    const float r = rintf(d);                      /* nearest, ties to even */
                    q = !(r > 0.0f) ? 0u : r >= (float)qmax ? (uint32_t)qmax : (uint32_t)r;
                }
                put_code(row, k, bits, q);
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * FP quantizer (wh-iron kernel-op coverage audit, "fp_quantized (fp4/fp8
 * quant + dequant)" row: a per-group max scale and mantissa rounding, exact
 * for fp8 normals and subnormals, saturating with no NaN or infinity; Track 1
 * format table for the block sizes and scale types).  The pages give no
 * formula for the scale; the reading here:
 *   MXFP4 / MXFP8-E4M3, blocks of 32: the E8M0 byte is
 *     clamp(floor(log2(amax)) - emax + 127, 0, 254)   (emax 2 for E2M1, 8 for
 *     E4M3; byte 0 when amax is 0), and element d = w * 2^(127 - byte);
 *   NVFP4, blocks of 16, FP32 global g > 0: the E4M3 scale is the nearest E4M3
 *     to t = amax / (6 * g) (fp32 operations), and d = w / (scale * g) (fp32
 *     operations; d = 0 when the scale is 0).
 * Every code is the element whose value is nearest to |d| (exact distances
 * below the largest element), ties to the even code, and the largest finite
 * element from there up (saturation); the sign bit is set for d < 0.  Codes are found by trying every element value, not
 * by arithmetic on the bits.  Rows [n0, n1).
 * ------------------------------------------------------------------------- */
/* Nearest E2M1 magnitude code (0..7) to a >= 0, ties to even, saturating:
 * from the largest element up the code is the largest (the distances of a
 * huge a to the elements would round to the same fp64 value). */
static uint32_t nearest_e2m1(double a) {
    if (a >= oracle_e2m1(7)) return 7;
    uint32_t best = 0;
    double bd = INFINITY;
    for (uint32_t c = 0; c < 8; ++c) {
        double dd = fabs(oracle_e2m1(c) - a);
        if (dd < bd || (dd == bd && (c & 1u) == 0)) { bd = dd; best = c; }
    }
    return best;
}

/* Nearest finite E4M3 magnitude code (0..126) to a >= 0, ties to even,
 * saturating at 448 as above. */
static uint32_t nearest_e4m3(double a) {
    if (a >= oracle_e4m3(126)) return 126;
    uint32_t best = 0;
    double bd = INFINITY;
    for (uint32_t c = 0; c < 127; ++c) {
        double dd = fabs(oracle_e4m3(c) - a);
        if (dd < bd || (dd == bd && (c & 1u) == 0)) { bd = dd; best = c; }
    }
    return best;
}

uint32_t oracle_nearest_e2m1(double a) { return nearest_e2m1(a); }
uint32_t oracle_nearest_e4m3(double a) { return nearest_e4m3(a); }

void oracle_quantize_fp(const void* w, uint8_t* wq, uint8_t* scales, float global, long long N, long long K,
                        int mode, int dtype, long long n0, long long n1) {
    (void)N;
    const int fp8 = mode == OR_MXFP8, nv = mode == OR_NVFP4;
    const int blk = nv ? 16 : 32;
    const long long rb = fp8 ? K : K / 2;
    for (long long n = n0; n < n1; ++n) {
        uint8_t* row = wq + n * rb;
        memset(row, 0, (size_t)rb);
        for (long long b0 = 0; b0 < K; b0 += blk) {
            float amax = 0.0f;
            for (long long k = b0; k < b0 + blk; ++k) {
                float a = fabsf(load_f32(w, (size_t)(n * K + k), dtype));
                if (a > amax) amax = a;
            }
            const size_t si = (size_t)(n * (K / blk) + b0 / blk);
            float sT = 0.0f;                 /* NVFP4 scale value */
            double mul = 0.0;                /* MX: 2^(127 - byte) */
            if (nv) {
                const float t = amax / (6.0f * global);              /* fp32, fp32 */
                const uint32_t sc = nearest_e4m3((double)t);
                scales[si] = (uint8_t)sc;
                sT = (float)oracle_e4m3(sc);
            } else {
                int byte = 0;
                if (amax > 0.0f) {
                    int e;
                    frexp((double)amax, &e);                          /* amax = f * 2^e, f in [0.5, 1) */
                    int x = (e - 1) - (fp8 ? 8 : 2) + 127;
                    byte = x < 0 ? 0 : x > 254 ? 254 : x;
                }
                scales[si] = (uint8_t)byte;
                mul = ldexp(1.0, 127 - byte);
            }
            for (long long k = b0; k < b0 + blk; ++k) {
                const float v = load_f32(w, (size_t)(n * K + k), dtype);
                double d;
                if (nv) d = sT == 0.0f ? 0.0 : (double)(v / (sT * global));   /* fp32, fp32 */
                else d = (double)v * mul;                                      /* exact */
                uint32_t code;
                if (fp8) code = nearest_e4m3(fabs(d)) | (d < 0 ? 0x80u : 0u);
                else code = nearest_e2m1(fabs(d)) | (d < 0 ? 0x8u : 0u);
                if (fp8) row[k] = (uint8_t)code;
                else row[k / 2] |= (uint8_t)(code << (4 * (k % 2)));
            }
        }
    }
}
