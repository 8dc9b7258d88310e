/*
 * tint4_oracle.c -- plain, slow CPU oracle for the packed-INT4 ConvRot
 * quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load or call this code.  The
 * product (the CUDA library) never links, loads or calls it, and the two share
 * no code: no headers, helpers, tables or constants.
 *
 * What it restates (page titles and sections):
 *  - "ComfyUI-INT-Crush", section "Forward Pass": rotate the activations
 *    (Hadamard, rot_size), then quantize weights and activations and run the
 *    GEMM.  Section "Inference > INT4 > CUDA backend": INT4 weights are
 *    unpacked to INT8 and fed to an INT8 GEMM with fused dequant.  Section
 *    "Inference > INT4 > Triton backend": activations are quantized
 *    dynamically.  Section "Inference > INT4 > PyTorch backend": the slow path
 *    is full dequant followed by a plain linear; this file is that slow path
 *    restated on the integer codes.  Section "Weight Format": INT4 weights are
 *    uint8 with two values per byte.
 *  - "feat: packed int4 convrot model loading and dispatch" (stable-diffusion.cpp
 *    #2010), section "Summary": packed nibbles are kept as they are, about half
 *    a byte per weight, with row scales beside them; convrot group sizes 64
 *    and 256.
 *  - "TINT4 v1.2 -- torchao INT4 量化推理 for ComfyUI", sections "量化方案" and
 *    "参数选择指南": Hadamard (QuaRot) rotation and the group sizes; section
 *    "v1.1 新特性 > 5": the W4A16 layer keeps _qdata/_scale/_zp, i.e. uint4
 *    codes with a scale and a zero point per group.
 *
 * The pages fix none of the arithmetic below (matrix, rounding, nibble order,
 * scale precision).  The readings taken here, each stated where it is used:
 *  - H_g is the Sylvester Hadamard matrix in natural order, scaled by 1/sqrt(g)
 *    so that it is orthonormal.  g is a power of four, so 1/sqrt(g) is a power
 *    of two and the scaling is exact.
 *  - The rotation decides the quantized codes, so it is computed in fp32 (the
 *    kernel's precision) with the fast Walsh-Hadamard transform in its
 *    textbook stage order (span 1, 2, 4, ... g/2), butterfly (a, b) ->
 *    (a + b, a - b), then the exact 1/sqrt(g) scaling.
 *  - Scales: absmax / 7 (int4) or absmax / 127 (int8), fp32 IEEE division.
 *    Codes: round half to even of v / s (fp32 IEEE division), clamped to
 *    [-7, 7] or [-127, 127].  A zero row has scale 0 and all codes 0.
 *  - Packing: byte j of a row holds code 2j in its low nibble and code 2j+1 in
 *    its high nibble (two's complement nibbles).
 *  - Epilogue and W4A16 are plain floating point with no decision, so they are
 *    evaluated in fp64 and rounded once to bf16 (round to nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG -1

/* ------------------------------------------------------------------------ */
/* bf16 <-> float / double                                                  */
/* ------------------------------------------------------------------------ */

static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to the nearest bf16 (ties to even), returning its bits.
 * bf16 has 8 significant bits and the fp32 exponent range; below 2^-126 the
 * grid is the subnormal spacing 2^-133. */
static uint16_t double_to_bf16_bits(double v) {
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else if (a < ldexp(1.0, -126)) {
        r = nearbyint(a * ldexp(1.0, 133)) * ldexp(1.0, -133);
    } else {
        int e;
        double m = frexp(a, &e);             /* a = m * 2^e, m in [0.5, 1) */
        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);
    }
    float f = (float)r;                      /* exact: r is on the bf16 grid */
    if (v < 0) f = -f;
    uint32_t u;
    memcpy(&u, &f, 4);  /* an out-of-range r became +-inf, whose top half is bf16 inf */
    return (uint16_t)(u >> 16);
}

/* Round a float to the nearest IEEE fp16 number (ties to even), returned as
 * the float of the same value (every fp16 value is exact in fp32).  fp16 has
 * 11 significant bits and exponents -14..15; below 2^-14 the grid is the
 * subnormal spacing 2^-24; a result above the largest finite value 65504
 * (that is, from 65520 on) is infinity.  "ComfyUI-INT-Crush", "Weight
 * Format": the stored weight scales are fp16. */
static float round_to_f16(float v) {
    if (isnan(v)) return v;
    double a = fabs((double)v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else if (a < ldexp(1.0, -14)) {
        r = nearbyint(a * ldexp(1.0, 24)) * ldexp(1.0, -24);
    } else {
        int e;
        double m = frexp(a, &e);              /* a = m * 2^e, m in [0.5, 1) */
        r = ldexp(nearbyint(ldexp(m, 11)), e - 11);
    }
    if (r > 65504.0) r = INFINITY;
    return (float)copysign(r, (double)v);
}

int oracle_round_f16(const float* v, long n, float* out) {
    if ((!v || !out) && n > 0) return ORACLE_BAD_ARG;
    for (long i = 0; i < n; ++i) out[i] = round_to_f16(v[i]);
    return ORACLE_OK;
}

static int is_power_of_four(int g) {
    if (g < 4) return 0;
    while (g > 1) {
        if (g % 4) return 0;
        g /= 4;
    }
    return 1;
}

/* ------------------------------------------------------------------------ */
/* Hadamard matrix and the fast Walsh-Hadamard transform                    */
/* ------------------------------------------------------------------------ */

/* Dense orthonormal Sylvester Hadamard matrix, row-major g x g, fp64:
 * H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]], then scaled by 1/sqrt(g). */
int oracle_hadamard(int g, double* H) {
    if (g < 1 || (g & (g - 1)) || !H) return ORACLE_BAD_ARG;
    H[0] = 1.0;
    for (int n = 1; n < g; n *= 2) {
        /* grow the n x n block in the top-left corner to 2n x 2n, in place */
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                double h = H[(long)i * g + j];
                H[(long)i * g + j + n] = h;
                H[(long)(i + n) * g + j] = h;
                H[(long)(i + n) * g + j + n] = -h;
            }
    }
    double s = 1.0 / sqrt((double)g);
    for (long i = 0; i < (long)g * g; ++i) H[i] *= s;
    return ORACLE_OK;
}

/* In-place orthonormal FWHT of one block of g fp32 values.  Stage spans go
 * 1, 2, 4, ..., g/2; each butterfly replaces (a, b) = (v[j], v[j+h]) with
 * (a + b, a - b).  Then every value is multiplied by 1/sqrt(g) = 2^-log4(g),
 * which is exact. */
static void fwht_f32_block(float* v, int g) {
    for (int h = 1; h < g; h *= 2)
        for (int i = 0; i < g; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    int log4 = 0;
    for (int t = g; t > 1; t /= 4) ++log4;
    float s = ldexpf(1.0f, -log4);
    for (int j = 0; j < g; ++j) v[j] *= s;
}

int oracle_fwht_f32(float* v, int g) {
    if (!v || !is_power_of_four(g)) return ORACLE_BAD_ARG;
    fwht_f32_block(v, g);
    return ORACLE_OK;
}

/* Rotate every length-g block along K of every row, in place (fp32).
 * g == 0 means no rotation. */
int oracle_rotate_rows_f32(float* rows, long nrows, int K, int g) {
    if (!rows || nrows < 0 || K <= 0) return ORACLE_BAD_ARG;
    if (g == 0) return ORACLE_OK;
    if (!is_power_of_four(g) || K % g) return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < nrows; ++r)
        for (int b = 0; b < K; b += g) fwht_f32_block(rows + r * (long)K + b, g);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Symmetric per-row quantization                                           */
/* ------------------------------------------------------------------------ */

/* One row of K fp32 values -> codes in [-qmax, qmax] and one fp32 scale.
 * scale = absmax / qmax; code = clamp(rne(v / scale)); zero row -> scale 0,
 * codes 0. */
static void quantize_row_s(const float* v, int K, int qmax, int s16, int8_t* q, float* scale) {
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
        float a = fabsf(v[k]);
        if (a > amax) amax = a;
    }
    float s = amax / (float)qmax;
    /* fp16 storage: the codes are taken against the stored scale */
    if (s16) s = round_to_f16(s);
    *scale = s;
    for (int k = 0; k < K; ++k) {
        int c = 0;
        if (s > 0.0f) {
            float t = rintf(v[k] / s);   /* default rounding mode: to nearest even */
            if (t > (float)qmax) t = (float)qmax;
            if (t < (float)-qmax) t = (float)-qmax;
            c = (int)t;
        }
        q[k] = (int8_t)c;
    }
}

static void quantize_row(const float* v, int K, int qmax, int8_t* q, float* scale) {
    quantize_row_s(v, K, qmax, 0, q, scale);
}

/* ------------------------------------------------------------------------ */
/* Nibble packing                                                           */
/* ------------------------------------------------------------------------ */

/* codes int8 [rows, K] (values in [-8, 7]) -> uint8 [rows, K/2]:
 * byte j = (code[2j] & 0xF) | ((code[2j+1] & 0xF) << 4). */
int oracle_pack_int4(const int8_t* q, long rows, int K, uint8_t* packed) {
    if (!q || !packed || rows < 0 || K <= 0 || K % 2) return ORACLE_BAD_ARG;
    for (long r = 0; r < rows; ++r)
        for (int j = 0; j < K / 2; ++j) {
            uint8_t lo = (uint8_t)(q[r * K + 2 * j] & 0xF);
            uint8_t hi = (uint8_t)(q[r * K + 2 * j + 1] & 0xF);
            packed[r * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
    return ORACLE_OK;
}

/* uint8 [rows, K/2] -> int8 codes [rows, K], each nibble read as a 4-bit
 * two's complement number. */
int oracle_unpack_int4(const uint8_t* packed, long rows, int K, int8_t* q) {
    if (!q || !packed || rows < 0 || K <= 0 || K % 2) return ORACLE_BAD_ARG;
    for (long r = 0; r < rows; ++r)
        for (int j = 0; j < K / 2; ++j) {
            uint8_t b = packed[r * (K / 2) + j];
            int lo = b & 0xF, hi = b >> 4;
            q[r * K + 2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            q[r * K + 2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Offline weight preparation (twin of tint4_pack_weights)                  */
/* ------------------------------------------------------------------------ */

/* W fp32 [N, K] -> rotate each g-block along K -> per-row symmetric int4
 * codes in [-7, 7] with fp32 row scale -> packed uint8 [N, K/2].
 * codes (optional, may be NULL) receives the unpacked int8 codes [N, K]. */
int oracle_pack_weights(const float* W, int N, int K, int g, uint8_t* packed,
                        float* row_scale, int8_t* codes) {
    if (!W || !packed || !row_scale || N <= 0 || K <= 0 || K % 2) return ORACLE_BAD_ARG;
    if (g != 0 && (!is_power_of_four(g) || K % g)) return ORACLE_BAD_ARG;
    int bad = 0;
#pragma omp parallel
    {
        float* v = (float*)malloc(sizeof(float) * (size_t)K);
        int8_t* q = (int8_t*)malloc((size_t)K);
        if (!v || !q) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int n = 0; n < N; ++n) {
                memcpy(v, W + (long)n * K, sizeof(float) * (size_t)K);
                if (g) for (int b = 0; b < K; b += g) fwht_f32_block(v + b, g);
                quantize_row(v, K, 7, q, &row_scale[n]);
                oracle_pack_int4(q, 1, K, packed + (long)n * (K / 2));
                if (codes) memcpy(codes + (long)n * K, q, (size_t)K);
            }
        }
        free(v);
        free(q);
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* W8A8 weights ("ComfyUI-INT-Crush", "Inference > INT8": the INT8 path
 * multiplies int8 weights by int8 activations with int32 accumulation):
 * W fp32 [N, K] -> rotate each g-block along K -> per-row symmetric int8
 * codes in [-127, 127] [N, K] with an fp32 row scale absmax / 127. */
/* As oracle_quantize_weights_int8, with the row scale rounded to fp16 (and
 * the codes taken against that stored scale) when s16 != 0. */
int oracle_quantize_weights_int8_ex(const float* W, int N, int K, int g, int s16, int8_t* codes,
                                    float* row_scale);

int oracle_quantize_weights_int8(const float* W, int N, int K, int g, int8_t* codes,
                                 float* row_scale) {
    return oracle_quantize_weights_int8_ex(W, N, K, g, 0, codes, row_scale);
}

int oracle_quantize_weights_int8_ex(const float* W, int N, int K, int g, int s16, int8_t* codes,
                                    float* row_scale) {
    if (!W || !codes || !row_scale || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    if (g != 0 && (!is_power_of_four(g) || K % g)) return ORACLE_BAD_ARG;
    int bad = 0;
#pragma omp parallel
    {
        float* v = (float*)malloc(sizeof(float) * (size_t)K);
        if (!v) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int n = 0; n < N; ++n) {
                memcpy(v, W + (long)n * K, sizeof(float) * (size_t)K);
                if (g) for (int b = 0; b < K; b += g) fwht_f32_block(v + b, g);
                quantize_row_s(v, K, 127, s16, codes + (long)n * K, &row_scale[n]);
            }
        }
        free(v);
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Dynamic per-token activation quantization (twin of convrot_quantize_act) */
/* ------------------------------------------------------------------------ */

/* x bf16 bits [M, K] -> fp32 -> rotate each g-block -> per-token symmetric
 * codes: bits 8 -> int8 in [-127, 127]; bits 4 -> int4 in [-7, 7].
 * codes_i8 receives the unpacked codes [M, K] (always int8, one per value);
 * packed (optional, bits 4 only) receives uint8 [M, K/2]. */
int oracle_quantize_act(const uint16_t* x, int M, int K, int g, int bits,
                        int8_t* codes_i8, float* tok_scale, uint8_t* packed) {
    if (!x || !codes_i8 || !tok_scale || M < 0 || K <= 0 || K % 2) return ORACLE_BAD_ARG;
    if (bits != 8 && bits != 4) return ORACLE_BAD_ARG;
    if (g != 0 && (!is_power_of_four(g) || K % g)) return ORACLE_BAD_ARG;
    int qmax = bits == 8 ? 127 : 7;
    int bad = 0;
#pragma omp parallel
    {
        float* v = (float*)malloc(sizeof(float) * (size_t)K);
        if (!v) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int m = 0; m < M; ++m) {
                for (int k = 0; k < K; ++k) v[k] = bf16_bits_to_float(x[(long)m * K + k]);
                if (g) for (int b = 0; b < K; b += g) fwht_f32_block(v + b, g);
                quantize_row(v, K, qmax, codes_i8 + (long)m * K, &tok_scale[m]);
                if (bits == 4 && packed)
                    oracle_pack_int4(codes_i8 + (long)m * K, 1, K, packed + (long)m * (K / 2));
            }
        }
        free(v);
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Integer GEMM and epilogue                                                */
/* ------------------------------------------------------------------------ */

/* acc[m, n] = sum_k a[m, k] * w[n, k], exact integer arithmetic.  Returns
 * ORACLE_BAD_ARG if a sum does not fit in int32. */
int oracle_gemm_i32(const int8_t* a, const int8_t* w, int M, int N, int K, int32_t* acc) {
    if (!a || !w || !acc || M < 0 || N < 0 || K < 0) return ORACLE_BAD_ARG;
    int overflow = 0;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int k = 0; k < K; ++k) s += (int64_t)a[(long)m * K + k] * (int64_t)w[(long)n * K + k];
            if (s > INT32_MAX || s < INT32_MIN) {
#pragma omp atomic write
                overflow = 1;
            }
            acc[(long)m * N + n] = (int32_t)s;
        }
    return overflow ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* The same sum for an explicit list of (m, n) pairs: pairs[2i] = m,
 * pairs[2i+1] = n. */
int oracle_gemm_i32_sampled(const int8_t* a, const int8_t* w, int K, const int64_t* pairs,
                            long npairs, int32_t* out) {
    if (!a || !w || !pairs || !out || K < 0 || npairs < 0) return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < npairs; ++i) {
        const int8_t* ar = a + pairs[2 * i] * (long)K;
        const int8_t* wr = w + pairs[2 * i + 1] * (long)K;
        int64_t s = 0;
        for (int k = 0; k < K; ++k) s += (int64_t)ar[k] * (int64_t)wr[k];
        out[i] = (int32_t)s;
    }
    return ORACLE_OK;
}

/* Fused dequant, unrounded: y[m, n] = acc * s_tok[m] * s_row[n] (+ bias[n]),
 * evaluated in fp64.  bias may be NULL. */
int oracle_epilogue_f64(const int32_t* acc, const float* s_tok, const float* s_row,
                        const uint16_t* bias, int M, int N, double* y) {
    if (!acc || !s_tok || !s_row || !y || M < 0 || N < 0) return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double v = (double)acc[(long)m * N + n] * (double)s_tok[m] * (double)s_row[n];
            if (bias) v += (double)bf16_bits_to_float(bias[n]);
            y[(long)m * N + n] = v;
        }
    return ORACLE_OK;
}

/* Fused dequant to the layer's bf16 output: the fp64 value above, rounded
 * once to bf16 (nearest, ties to even). */
int oracle_epilogue(const int32_t* acc, const float* s_tok, const float* s_row,
                    const uint16_t* bias, int M, int N, uint16_t* y) {
    if (!acc || !s_tok || !s_row || !y || M < 0 || N < 0) return ORACLE_BAD_ARG;
    double* t = (double*)malloc(sizeof(double) * ((size_t)M * N + 1));
    if (!t) return ORACLE_BAD_ARG;
    int rc = oracle_epilogue_f64(acc, s_tok, s_row, bias, M, N, t);
    for (long i = 0; rc == ORACLE_OK && i < (long)M * N; ++i) y[i] = double_to_bf16_bits(t[i]);
    free(t);
    return rc;
}

/* Epilogue for a list of (m, n) pairs with their accumulators, unrounded. */
int oracle_epilogue_sampled_f64(const int32_t* acc, const float* s_tok, const float* s_row,
                                const uint16_t* bias, const int64_t* pairs, long npairs,
                                double* y) {
    if (!acc || !s_tok || !s_row || !pairs || !y || npairs < 0) return ORACLE_BAD_ARG;
    for (long i = 0; i < npairs; ++i) {
        long m = pairs[2 * i], n = pairs[2 * i + 1];
        double v = (double)acc[i] * (double)s_tok[m] * (double)s_row[n];
        if (bias) v += (double)bf16_bits_to_float(bias[n]);
        y[i] = v;
    }
    return ORACLE_OK;
}

/* ... and rounded to bf16. */
int oracle_epilogue_sampled(const int32_t* acc, const float* s_tok, const float* s_row,
                            const uint16_t* bias, const int64_t* pairs, long npairs,
                            uint16_t* y) {
    if (!y || npairs < 0) return ORACLE_BAD_ARG;
    double* t = (double*)malloc(sizeof(double) * ((size_t)npairs + 1));
    if (!t) return ORACLE_BAD_ARG;
    int rc = oracle_epilogue_sampled_f64(acc, s_tok, s_row, bias, pairs, npairs, t);
    for (long i = 0; rc == ORACLE_OK && i < npairs; ++i) y[i] = double_to_bf16_bits(t[i]);
    free(t);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Whole W4A8 / W4A4 linear (twin of convrot_w4a8_linear / ..._w4a4_...)    */
/* ------------------------------------------------------------------------ */

/* y = (Q_act(rot(x)) . unpack(w_packed)^T) * s_tok * s_row (+ bias), unrounded
 * (fp64).  act_bits 8 or 4; g the rotation group (0: none).  Scratch is
 * allocated here. */
int oracle_convrot_linear_f64(const uint16_t* x, const uint8_t* w_packed, const float* row_scale,
                              const uint16_t* bias, int M, int N, int K, int g, int act_bits,
                              double* y) {
    if (!x || !w_packed || !row_scale || !y || M < 0 || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    int8_t* qa = (int8_t*)malloc((size_t)M * K + 1);
    int8_t* qw = (int8_t*)malloc((size_t)N * K + 1);
    float* st = (float*)malloc(sizeof(float) * (size_t)M + 4);
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)M * N + 4);
    int rc = ORACLE_BAD_ARG;
    if (qa && qw && st && acc) {
        rc = oracle_quantize_act(x, M, K, g, act_bits, qa, st, NULL);
        if (rc == ORACLE_OK) rc = oracle_unpack_int4(w_packed, N, K, qw);
        if (rc == ORACLE_OK) rc = oracle_gemm_i32(qa, qw, M, N, K, acc);
        if (rc == ORACLE_OK) rc = oracle_epilogue_f64(acc, st, row_scale, bias, M, N, y);
    }
    free(qa);
    free(qw);
    free(st);
    free(acc);
    return rc;
}

/* The layer's bf16 output: the value above rounded once to bf16. */
int oracle_convrot_linear(const uint16_t* x, const uint8_t* w_packed, const float* row_scale,
                          const uint16_t* bias, int M, int N, int K, int g, int act_bits,
                          uint16_t* y) {
    if (!y || M < 0 || N <= 0) return ORACLE_BAD_ARG;
    double* t = (double*)malloc(sizeof(double) * ((size_t)M * N + 1));
    if (!t) return ORACLE_BAD_ARG;
    int rc = oracle_convrot_linear_f64(x, w_packed, row_scale, bias, M, N, K, g, act_bits, t);
    for (long i = 0; rc == ORACLE_OK && i < (long)M * N; ++i) y[i] = double_to_bf16_bits(t[i]);
    free(t);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* W4A16 group-wise asymmetric linear (twin of w4a16_gemv_gemm)             */
/* ------------------------------------------------------------------------ */

/* y[m, n] = sum_k x[m, k] * (q[n, k] - z[n, k/G]) * s[n, k/G], unrounded, with
 * q uint4 packed low-first in uint8 [N, K/2], s bf16 [N, K/G], z uint8
 * [N, K/G] holding 0..15.  fp64 accumulation. */
int oracle_w4a16_f64(const uint16_t* x, const uint8_t* q, const uint16_t* s, const uint8_t* z,
                     int M, int N, int K, int G, double* y) {
    if (!x || !q || !s || !z || !y || M < 0 || N < 0 || K <= 0 || G <= 0 || K % G || K % 2)
        return ORACLE_BAD_ARG;
    int ng = K / G;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        for (int m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) {
                uint8_t b = q[(long)n * (K / 2) + k / 2];
                int code = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
                double w = ((double)code - (double)z[(long)n * ng + k / G]) *
                           (double)bf16_bits_to_float(s[(long)n * ng + k / G]);
                acc += (double)bf16_bits_to_float(x[(long)m * K + k]) * w;
            }
            y[(long)m * N + n] = acc;
        }
    return ORACLE_OK;
}

/* The 16-bit unpack + 16-bit GEMM form ("ComfyUI-INT-Crush", "Inference >
 * INT4 > Triton backend": W4A16 widens the INT4 weights to 16 bits and runs a
 * 16-bit GEMM): every weight is first dequantized to the bf16 number nearest
 * to (q - z) * s (the product itself is exact in double), then
 * y[m, n] = sum_k x[m, k] * w[n, k] in fp64, unrounded. */
int oracle_w4a16_dequant_f64(const uint16_t* x, const uint8_t* q, const uint16_t* s,
                             const uint8_t* z, int M, int N, int K, int G, double* y) {
    if (!x || !q || !s || !z || !y || M < 0 || N < 0 || K <= 0 || G <= 0 || K % G || K % 2)
        return ORACLE_BAD_ARG;
    int ng = K / G;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int n = 0; n < N; ++n) {
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
        if (!w) {
            bad = 1;
            continue;
        }
        for (int k = 0; k < K; ++k) {
            uint8_t b = q[(long)n * (K / 2) + k / 2];
            int code = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
            double exact = ((double)code - (double)z[(long)n * ng + k / G]) *
                           (double)bf16_bits_to_float(s[(long)n * ng + k / G]);
            w[k] = (double)bf16_bits_to_float(double_to_bf16_bits(exact));
        }
        for (int m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += (double)bf16_bits_to_float(x[(long)m * K + k]) * w[k];
            y[(long)m * N + n] = acc;
        }
        free(w);
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* The W4A16 weights themselves, fp64 [N, K]: w = (q - z) * s exactly
 * (widen = 0), or that product rounded once to the nearest bf16 (widen = 1,
 * the 16-bit unpack form above).  A dense matrix product of x with these
 * gives the two forms of the layer for large shapes. */
int oracle_w4a16_weights_f64(const uint8_t* q, const uint16_t* s, const uint8_t* z, int N, int K,
                             int G, int widen, double* w) {
    if (!q || !s || !z || !w || N < 0 || K <= 0 || G <= 0 || K % G || K % 2) return ORACLE_BAD_ARG;
    int ng = K / G;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            uint8_t b = q[(long)n * (K / 2) + k / 2];
            int code = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
            double exact = ((double)code - (double)z[(long)n * ng + k / G]) *
                           (double)bf16_bits_to_float(s[(long)n * ng + k / G]);
            w[(long)n * K + k] =
                widen ? (double)bf16_bits_to_float(double_to_bf16_bits(exact)) : exact;
        }
    return ORACLE_OK;
}

/* The same, rounded once to bf16: the layer's output. */
int oracle_w4a16(const uint16_t* x, const uint8_t* q, const uint16_t* s, const uint8_t* z,
                 int M, int N, int K, int G, uint16_t* y) {
    if (!y || M < 0 || N < 0) return ORACLE_BAD_ARG;
    double* t = (double*)malloc(sizeof(double) * ((size_t)M * N + 1));
    if (!t) return ORACLE_BAD_ARG;
    int rc = oracle_w4a16_f64(x, q, s, z, M, N, K, G, t);
    for (long i = 0; rc == ORACLE_OK && i < (long)M * N; ++i) y[i] = double_to_bf16_bits(t[i]);
    free(t);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Group-wise W4A8 weights and GEMM                                          */
/* ------------------------------------------------------------------------ */

/* "ComfyUI-INT-Crush", "Weight Format": the INT4 weight scales have one value
 * per output row and K group ([out, num_groups]).  stable-diffusion.cpp
 * "feat: packed int4 convrot model loading and dispatch", "Summary": an
 * asymmetric W4A8 format (asym_w4a8_int8) next to the symmetric one.
 * Readings (the pages fix none of this arithmetic):
 *  - a weight group is G consecutive K values of one row, after the same
 *    block rotation as the per-row format; its scale is fp32;
 *  - symmetric: the per-row rule applied to the group: s = absmax / 7 and
 *    q = clamp(rne(v / s), -7, 7), stored as two's complement nibbles;
 *  - asymmetric: the group's range widened to contain 0, lo = min(0, min v),
 *    hi = max(0, max v); s = (hi - lo) / 15; zero point z = rne(-lo / s),
 *    clamped to [0, 15]; q = clamp(rne(v / s) + z, 0, 15), stored as plain
 *    4-bit numbers; the weight the codes stand for is s * (q - z);
 *  - an all-zero group has s = 0, z = 0 and q = 0;
 *  - all of it in fp32 with IEEE division and round half to even (the codes
 *    are decisions, taken in the kernel's precision). */
static void quantize_group_asym(const float* v, int G, int s16, int8_t* q, float* scale,
                                uint8_t* zero) {
    float lo = 0.0f, hi = 0.0f;
    for (int k = 0; k < G; ++k) {
        if (v[k] < lo) lo = v[k];
        if (v[k] > hi) hi = v[k];
    }
    float s = (hi - lo) / 15.0f;
    if (s16) s = round_to_f16(s);   /* the zero point and codes use the stored scale */
    int z = 0;
    if (s > 0.0f) {
        float t = rintf(-lo / s);
        if (t < 0.0f) t = 0.0f;
        if (t > 15.0f) t = 15.0f;
        z = (int)t;
    }
    *scale = s;
    *zero = (uint8_t)z;
    for (int k = 0; k < G; ++k) {
        int c = 0;
        if (s > 0.0f) {
            c = (int)rintf(v[k] / s) + z;
            if (c < 0) c = 0;
            if (c > 15) c = 15;
        }
        q[k] = (int8_t)c;
    }
}

/* W fp32 [N, K] -> rotate each g-block along K -> group-wise int4 codes with
 * scale fp32 [N, K/G] (and zero uint8 [N, K/G] when asym) -> packed uint8
 * [N, K/2], byte j holding code 2j in its low nibble.  codes (optional)
 * receives the codes as int8 [N, K]: signed for the symmetric form, 0..15 for
 * the asymmetric one.  zero may be NULL when asym == 0. */
/* As oracle_pack_weights_groupwise, with every group scale rounded to fp16
 * (and the zero points and codes taken against that stored scale) when
 * s16 != 0; scale then holds the fp16 values as floats. */
int oracle_pack_weights_groupwise_ex(const float* W, int N, int K, int g, int G, int asym, int s16,
                                     uint8_t* packed, float* scale, uint8_t* zero, int8_t* codes);

int oracle_pack_weights_groupwise(const float* W, int N, int K, int g, int G, int asym,
                                  uint8_t* packed, float* scale, uint8_t* zero, int8_t* codes) {
    return oracle_pack_weights_groupwise_ex(W, N, K, g, G, asym, 0, packed, scale, zero, codes);
}

int oracle_pack_weights_groupwise_ex(const float* W, int N, int K, int g, int G, int asym, int s16,
                                     uint8_t* packed, float* scale, uint8_t* zero, int8_t* codes) {
    if (!W || !packed || !scale || (asym && !zero) || N <= 0 || K <= 0 || K % 2 || G <= 0 ||
        G % 2 || K % G)
        return ORACLE_BAD_ARG;
    if (g != 0 && (!is_power_of_four(g) || K % g)) return ORACLE_BAD_ARG;
    const int ng = K / G;
    int bad = 0;
#pragma omp parallel
    {
        float* v = (float*)malloc(sizeof(float) * (size_t)K);
        int8_t* q = (int8_t*)malloc((size_t)K);
        if (!v || !q) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int n = 0; n < N; ++n) {
                memcpy(v, W + (long)n * K, sizeof(float) * (size_t)K);
                if (g) for (int b = 0; b < K; b += g) fwht_f32_block(v + b, g);
                for (int j = 0; j < ng; ++j) {
                    if (asym)
                        quantize_group_asym(v + (long)j * G, G, s16, q + (long)j * G,
                                            &scale[(long)n * ng + j], &zero[(long)n * ng + j]);
                    else
                        quantize_row_s(v + (long)j * G, G, 7, s16, q + (long)j * G,
                                       &scale[(long)n * ng + j]);
                }
                oracle_pack_int4(q, 1, K, packed + (long)n * (K / 2));
                if (codes) memcpy(codes + (long)n * K, q, (size_t)K);
            }
        }
        free(v);
        free(q);
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* Code of weight (n, k): the nibble read as two's complement (symmetric) or
 * as a plain 4-bit number (asymmetric). */
static int groupwise_code(const uint8_t* packed, int K, int n, int k, int asym) {
    uint8_t b = packed[(long)n * (K / 2) + k / 2];
    int c = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
    if (!asym && c >= 8) c -= 16;
    return c;
}

/* One output of the group-wise W4A8 GEMM ("ComfyUI-INT-Crush", "Inference >
 * INT4 > CUDA backend": integer GEMM, then dequant; "Weight Format": one
 * scale per row and group): with the group's integer sum
 *   p_j = sum_{k in group j} a[m, k] * (q[n, k] - z[n, j])     (exact),
 *   y = s_tok[m] * sum_j s[n, j] * p_j (+ bias[n])              (fp64),
 * and mag = |s_tok[m]| * sum_j |s[n, j] * p_j| + |bias[n]|, the size of the
 * terms a floating-point evaluation adds up. */
static void groupwise_one(const int8_t* a, const float* tok_scale, const uint8_t* packed,
                          const float* scale, const uint8_t* zero, const uint16_t* bias, int N,
                          int K, int G, int m, int n, double* y, double* mag) {
    const int ng = K / G;
    const int asym = zero != NULL;
    double acc = 0.0, sum_abs = 0.0;
    for (int j = 0; j < ng; ++j) {
        const int z = asym ? zero[(long)n * ng + j] : 0;
        long p = 0;
        for (int k = j * G; k < (j + 1) * G; ++k)
            p += (long)a[(long)m * K + k] * (groupwise_code(packed, K, n, k, asym) - z);
        const double t = (double)scale[(long)n * ng + j] * (double)p;
        acc += t;
        sum_abs += fabs(t);
    }
    const double b = bias ? (double)bf16_bits_to_float(bias[n]) : 0.0;
    *y = acc * (double)tok_scale[m] + b;
    if (mag) *mag = fabs((double)tok_scale[m]) * sum_abs + fabs(b);
    (void)N;
}

/* y fp64 [M, N] (unrounded) and, optionally, mag fp64 [M, N]; a int8 [M, K],
 * zero NULL for the symmetric form. */
int oracle_gemm_groupwise_f64(const int8_t* a, const float* tok_scale, const uint8_t* packed,
                              const float* scale, const uint8_t* zero, const uint16_t* bias,
                              int M, int N, int K, int G, double* y, double* mag) {
    if (!a || !tok_scale || !packed || !scale || !y || M < 0 || N < 0 || K <= 0 || K % 2 ||
        G <= 0 || K % G)
        return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        for (int m = 0; m < M; ++m)
            groupwise_one(a, tok_scale, packed, scale, zero, bias, N, K, G, m, n,
                          &y[(long)m * N + n], mag ? &mag[(long)m * N + n] : NULL);
    return ORACLE_OK;
}

/* The same for a list of (m, n) pairs: pairs[2i] = m, pairs[2i + 1] = n. */
int oracle_gemm_groupwise_sampled_f64(const int8_t* a, const float* tok_scale,
                                      const uint8_t* packed, const float* scale,
                                      const uint8_t* zero, const uint16_t* bias, int M, int N,
                                      int K, int G, const int64_t* pairs, long npairs, double* y,
                                      double* mag) {
    if (!a || !tok_scale || !packed || !scale || !pairs || !y || npairs < 0 || K <= 0 ||
        K % 2 || G <= 0 || K % G)
        return ORACLE_BAD_ARG;
    for (long i = 0; i < npairs; ++i)
        if (pairs[2 * i] < 0 || pairs[2 * i] >= M || pairs[2 * i + 1] < 0 || pairs[2 * i + 1] >= N)
            return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < npairs; ++i)
        groupwise_one(a, tok_scale, packed, scale, zero, bias, N, K, G, (int)pairs[2 * i],
                      (int)pairs[2 * i + 1], &y[i], mag ? &mag[i] : NULL);
    return ORACLE_OK;
}

/* Round an array of doubles to bf16 bits (nearest, ties to even). */
int oracle_round_bf16(const double* v, long n, uint16_t* out) {
    if (!v || !out || n < 0) return ORACLE_BAD_ARG;
    for (long i = 0; i < n; ++i) out[i] = double_to_bf16_bits(v[i]);
    return ORACLE_OK;
}

/* fp64 -> bf16 rounding exposed for the tests of the rounding itself. */
uint16_t oracle_double_to_bf16(double v) { return double_to_bf16_bits(v); }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
