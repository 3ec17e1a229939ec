/*
 * Host oracle for W4A16 weight-only round-to-nearest (RTN) quantization, and
 * for its 8-bit form W8A16 (the section near the end of this file).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this code.  It shares no source,
 * header, table or helper with the CUDA library; the CUDA path never calls it.
 *
 * Plain scalar C, one element at a time, in the order the pages describe the
 * method.  Floating point follows IEEE-754 binary32 (float) for the quantizer
 * arithmetic and binary64 (double) for the reference matmul.  Build without
 * -ffast-math and with -ffp-contract=off so that no multiply-add is fused.
 *
 * Pages followed (titles as published):
 *  [P3] "量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）", §二 量化的数学本质:
 *       q = round(x/s) + z,  x ≈ s·(q − z);  absmax: s = max|x| / (2^(b−1) − 1);
 *       granularity table: per-group = one scale per 128 elements.
 *  [P4] "推理优化中“用精度换性能“的核心技术：量化":
 *       §2.2 INT4 holds [−8, 7] or [0, 15];
 *       §2.3 x_int = round(x_float / s) + z,  x̂_float = (x_int − z) × s;
 *       §3.3 symmetric s = max|x| / max_int, z = 0;
 *            asymmetric s = (max(x) − min(x)) / 255 (INT8; 15 for INT4),
 *            z = round(−min(x) / s);
 *       §3.4 group-wise: group_size 128 shares one 16-bit scale and an
 *            optional 16-bit zero point (4 + 32/128 = 4.25 bits per weight);
 *       §3.2 weight-only: load INT4 → dequantize to FP16/BF16 → matmul with
 *            16-bit activations.
 *  [P5] "LLM 量化中 W4A16 表示什么…｜蚂蚁集团 C/C++面经解析", 显存收益主要来自权重:
 *       the INT4 body costs 0.5 byte per weight (two codes per byte).
 *
 * Readings where the pages are silent, ambiguous or garbled:
 *  R1 round() is round-half-to-even in binary32 (rintf under FE_TONEAREST).
 *  R2 s is computed in binary32, rounded to bf16, and z and q are computed with
 *     the stored bf16 value of s.
 *  R3 codes are clamped to the INT4 range ([0,15] asym, [−8,7] sym).
 *  R4 the asymmetric range is widened to contain zero: mn = min(0, min x),
 *     mx = max(0, max x), so z lies in [0, 15] and 0 is on the grid.
 *  R5 a group whose s rounds to 0 (all zeros) gets z = 0 and q = 0.
 *  R6 sym codes are stored as 4-bit two's complement; zeros are written as 0.
 *  R7 code of element k = 2i is the low nibble of byte i, k = 2i+1 the high.
 *  R8 the dequantized weight is bf16_rn((q − z)·s): (q − z) is an exact
 *     integer, the product is exact in binary32, and one rounding to bf16.
 *  R9 groups run along K (input channels) of W[N, K].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------------
 * bf16 <-> binary32 / binary64.  bf16 is the upper half of a binary32
 * (1 sign, 8 exponent, 7 mantissa bits; [P4] §2.1).
 * ------------------------------------------------------------------------- */

float oracle_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 to the nearest bf16, ties to even. */
uint16_t oracle_f32_to_bf16_rn(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) {          /* NaN: keep it a quiet NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    }
    uint32_t keep_lsb = (u >> 16) & 1u;              /* lowest kept bit */
    u += 0x7fffu + keep_lsb;                         /* exact half rounds to even */
    return (uint16_t)(u >> 16);
}

/* Round a binary64 to the nearest bf16 with ONE rounding (no detour through
 * binary32), ties to even.  Used for the reference output bf16_rn(Y64). */
uint16_t oracle_f64_to_bf16_rn(double d) {
    if (isnan(d)) return 0x7fc0u;
    uint16_t sign = signbit(d) ? 0x8000u : 0u;
    double a = fabs(d);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7f80u);
    int e;
    (void)frexp(a, &e);                   /* a = m·2^e, m in [0.5, 1) */
    int quantum = e - 8;                  /* 8 significant bits for normals */
    if (quantum < -133) quantum = -133;   /* bf16 subnormal spacing 2^-133 */
    double r = nearbyint(ldexp(a, -quantum));   /* ties-to-even integer */
    double v = ldexp(r, quantum);
    const double bf16_max = 3.3895313892515355e38; /* (2 − 2^-7)·2^127 */
    if (v > bf16_max) return (uint16_t)(sign | 0x7f80u);
    float f = (float)v;                   /* exact: v has ≤ 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* ---------------------------------------------------------------------------
 * Quantization of one group ([P3] §二; [P4] §2.3, §3.3).
 * ------------------------------------------------------------------------- */

static float clamp_code(float r, float lo, float hi) {
    /* Clamp in binary32 before any integer conversion (R3). */
    if (r < lo) return lo;
    if (r > hi) return hi;
    return r;
}

/* Asymmetric group: s = (max − min)/15, z = round(−min/s), q = round(x/s) + z. */
void oracle_group_asym(const float* x, int64_t g, uint16_t* s_out, int32_t* z_out,
                       int32_t* q_out) {
    float mn = 0.0f, mx = 0.0f;                       /* R4: range contains 0 */
    for (int64_t i = 0; i < g; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    float s32 = (mx - mn) / 15.0f;                    /* 2^4 − 1 levels */
    uint16_t s_bits = oracle_f32_to_bf16_rn(s32);     /* R2 */
    float s = oracle_bf16_to_f32(s_bits);
    int32_t z = 0;
    if (s != 0.0f) {
        z = (int32_t)clamp_code(rintf(-mn / s), 0.0f, 15.0f);
    }
    for (int64_t i = 0; i < g; ++i) {
        int32_t q = 0;
        if (s != 0.0f) {                              /* R5 */
            float r = clamp_code(rintf(x[i] / s), -32.0f, 32.0f);
            q = (int32_t)r + z;
            if (q < 0) q = 0;
            if (q > 15) q = 15;
        }
        q_out[i] = q;
    }
    *s_out = s_bits;
    *z_out = z;
}

/* Symmetric (absmax) group: s = max|x| / 7, z = 0, q = round(x/s). */
void oracle_group_sym(const float* x, int64_t g, uint16_t* s_out, int32_t* q_out) {
    float amax = 0.0f;
    for (int64_t i = 0; i < g; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s32 = amax / 7.0f;                          /* 2^(4−1) − 1 */
    uint16_t s_bits = oracle_f32_to_bf16_rn(s32);
    float s = oracle_bf16_to_f32(s_bits);
    for (int64_t i = 0; i < g; ++i) {
        int32_t q = 0;
        if (s != 0.0f) {
            float r = clamp_code(rintf(x[i] / s), -32.0f, 32.0f);
            q = (int32_t)r;
            if (q < -8) q = -8;
            if (q > 7) q = 7;
        }
        q_out[i] = q;
    }
    *s_out = s_bits;
}

/* ---------------------------------------------------------------------------
 * Packing: two 4-bit codes per byte ([P5]; R6, R7).
 * ------------------------------------------------------------------------- */

void oracle_pack_codes(const int32_t* q, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n / 2; ++i) {
        uint32_t lo = (uint32_t)q[2 * i] & 0xFu;      /* two's complement nibble */
        uint32_t hi = (uint32_t)q[2 * i + 1] & 0xFu;
        out[i] = (uint8_t)(lo | (hi << 4));
    }
}

void oracle_unpack_codes(const uint8_t* packed, int64_t n, int32_t sym, int32_t* q) {
    for (int64_t k = 0; k < n; ++k) {
        uint8_t b = packed[k / 2];
        int32_t nib = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
        if (sym && nib >= 8) nib -= 16;              /* sign-extend 4-bit */
        q[k] = nib;
    }
}

/* ---------------------------------------------------------------------------
 * Whole-matrix quantize / dequantize.  W[N, K] row-major bf16 bits; groups of
 * g consecutive elements along K (R9).  packed[N, K/2], scales/zeros[N, K/g].
 * ------------------------------------------------------------------------- */

int oracle_quantize(const uint16_t* W, int64_t N, int64_t K, int64_t g, int32_t sym,
                    uint8_t* packed, uint16_t* scales, uint16_t* zeros) {
    if (N < 0 || K < 0 || g <= 0 || g % 2 != 0 || K % g != 0) return 1;
    const int64_t G = K / g;
    int failed = 0;
    #pragma omp parallel
    {
        float* xg = (float*)malloc((size_t)g * sizeof(float));
        int32_t* qg = (int32_t*)malloc((size_t)g * sizeof(int32_t));
        if (!xg || !qg) {
            #pragma omp atomic write
            failed = 1;
        }
        #pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            if (!xg || !qg) continue;
            for (int64_t j = 0; j < G; ++j) {
                const uint16_t* src = W + n * K + j * g;
                for (int64_t i = 0; i < g; ++i) xg[i] = oracle_bf16_to_f32(src[i]);
                uint16_t s_bits;
                int32_t z = 0;
                if (sym) {
                    oracle_group_sym(xg, g, &s_bits, qg);
                } else {
                    oracle_group_asym(xg, g, &s_bits, &z, qg);
                }
                scales[n * G + j] = s_bits;
                if (zeros) zeros[n * G + j] = oracle_f32_to_bf16_rn((float)z);
                oracle_pack_codes(qg, g, packed + n * (K / 2) + j * (g / 2));
            }
        }
        free(xg);
        free(qg);
    }
    return failed;
}

/* x̂ = bf16_rn((q − z)·s)   ([P4] §2.3; R8) */
static uint16_t dequant_one(int32_t q, int32_t z, float s) {
    float prod = (float)(q - z) * s;       /* exact: ≤ 5-bit integer × 8-bit significand */
    return oracle_f32_to_bf16_rn(prod);
}

int oracle_dequantize(const uint8_t* packed, const uint16_t* scales, const uint16_t* zeros,
                      int64_t N, int64_t K, int64_t g, int32_t sym, uint16_t* W_hat) {
    if (N < 0 || K < 0 || g <= 0 || g % 2 != 0 || K % g != 0) return 1;
    const int64_t G = K / g;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = packed[n * (K / 2) + k / 2];
            int32_t q = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
            if (sym && q >= 8) q -= 16;
            int64_t j = k / g;
            float s = oracle_bf16_to_f32(scales[n * G + j]);
            int32_t z = sym ? 0 : (int32_t)oracle_bf16_to_f32(zeros[n * G + j]);
            W_hat[n * K + k] = dequant_one(q, z, s);
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Reference matmul in binary64 on the dequantized weights:
 *   Y64[m, n] = Σ_k X[m, k] · x̂[n, k]
 * Every product of two bf16 values is exact in binary64; the sum runs in
 * increasing k.  ([P4] §3.2: dequantize, then multiply with 16-bit
 * activations.)
 * ------------------------------------------------------------------------- */

void oracle_gemm_f64(const uint16_t* X, int64_t M, int64_t K, const uint16_t* W_hat,
                     int64_t N, double* Y) {
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                acc += (double)oracle_bf16_to_f32(X[m * K + k]) *
                       (double)oracle_bf16_to_f32(W_hat[n * K + k]);
            }
            Y[m * N + n] = acc;
        }
    }
}

/* Same sum for a list of (m, n) output positions, dequantizing row n from the
 * packed form on the fly.  Used to check sampled outputs of large problems. */
int oracle_gemm_w4a16_sampled(const uint16_t* X, int64_t M, int64_t K, const uint8_t* packed,
                              const uint16_t* scales, const uint16_t* zeros, int64_t N,
                              int64_t g, int32_t sym, const int64_t* ms, const int64_t* ns,
                              int64_t count, double* out) {
    if (K % g != 0) return 1;
    const int64_t G = K / g;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0;
        if (m < 0 || m >= M || n < 0 || n >= N) {
            out[i] = NAN;
            continue;
        }
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = packed[n * (K / 2) + k / 2];
            int32_t q = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
            if (sym && q >= 8) q -= 16;
            int64_t j = k / g;
            float s = oracle_bf16_to_f32(scales[n * G + j]);
            int32_t z = sym ? 0 : (int32_t)oracle_bf16_to_f32(zeros[n * G + j]);
            uint16_t w = dequant_one(q, z, s);
            acc += (double)oracle_bf16_to_f32(X[m * K + k]) * (double)oracle_bf16_to_f32(w);
        }
        out[i] = acc;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * W8A16: 8-bit codes, one per byte.  [P4] §3.3 states the INT8 form itself:
 * asymmetric s = (max − min) / 255, z = round(−min / s); symmetric
 * s = max|x| / max_int with max_int = 2^(8−1) − 1 = 127 ([P3] §二 absmax,
 * b = 8).  [P2] 详细版 lists W8A16 beside W4A16 as a common scheme.
 * Readings, as for INT4 with the 8-bit ranges:
 *  R1, R2, R4, R5, R9 unchanged;
 *  R3' codes are clamped to [0, 255] (asym) or [−128, 127] (sym);
 *  R6' sym codes are stored as int8 two's complement, zeros written as 0;
 *  R7' code of element k is byte k of its row;
 *  R8' x̂ = bf16_rn((q − z)·s): |q − z| ≤ 255 has 8 significant bits, s has 8,
 *      so the product is exact in binary32 and is rounded once.
 *  Zero points are integers 0..255, exact in bf16 (8 significant bits).
 * ------------------------------------------------------------------------- */

/* Asymmetric 8-bit group: s = (max − min)/255, z = round(−min/s), q = round(x/s) + z. */
void oracle_group_asym8(const float* x, int64_t g, uint16_t* s_out, int32_t* z_out,
                        int32_t* q_out) {
    float mn = 0.0f, mx = 0.0f;                       /* R4: range contains 0 */
    for (int64_t i = 0; i < g; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    float s32 = (mx - mn) / 255.0f;                   /* 2^8 − 1 levels */
    uint16_t s_bits = oracle_f32_to_bf16_rn(s32);     /* R2 */
    float s = oracle_bf16_to_f32(s_bits);
    int32_t z = 0;
    if (s != 0.0f) {
        z = (int32_t)clamp_code(rintf(-mn / s), 0.0f, 255.0f);
    }
    for (int64_t i = 0; i < g; ++i) {
        int32_t q = 0;
        if (s != 0.0f) {                              /* R5 */
            float r = clamp_code(rintf(x[i] / s), -512.0f, 512.0f);
            q = (int32_t)r + z;
            if (q < 0) q = 0;
            if (q > 255) q = 255;
        }
        q_out[i] = q;
    }
    *s_out = s_bits;
    *z_out = z;
}

/* Symmetric (absmax) 8-bit group: s = max|x| / 127, z = 0, q = round(x/s). */
void oracle_group_sym8(const float* x, int64_t g, uint16_t* s_out, int32_t* q_out) {
    float amax = 0.0f;
    for (int64_t i = 0; i < g; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s32 = amax / 127.0f;                        /* 2^(8−1) − 1 */
    uint16_t s_bits = oracle_f32_to_bf16_rn(s32);
    float s = oracle_bf16_to_f32(s_bits);
    for (int64_t i = 0; i < g; ++i) {
        int32_t q = 0;
        if (s != 0.0f) {
            float r = clamp_code(rintf(x[i] / s), -512.0f, 512.0f);
            q = (int32_t)r;
            if (q < -128) q = -128;
            if (q > 127) q = 127;
        }
        q_out[i] = q;
    }
    *s_out = s_bits;
}

/* Code byte of element k (R6', R7'). */
static int32_t code8_of(const uint8_t* codes, int64_t idx, int32_t sym) {
    int32_t q = codes[idx];
    if (sym && q >= 128) q -= 256;                    /* int8 two's complement */
    return q;
}

/* W[N, K] -> codes[N, K] (one byte each), scales/zeros[N, K/g]. */
int oracle_quantize8(const uint16_t* W, int64_t N, int64_t K, int64_t g, int32_t sym,
                     uint8_t* codes, uint16_t* scales, uint16_t* zeros) {
    if (N < 0 || K < 0 || g <= 0 || K % g != 0) return 1;
    const int64_t G = K / g;
    int failed = 0;
    #pragma omp parallel
    {
        float* xg = (float*)malloc((size_t)g * sizeof(float));
        int32_t* qg = (int32_t*)malloc((size_t)g * sizeof(int32_t));
        if (!xg || !qg) {
            #pragma omp atomic write
            failed = 1;
        }
        #pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            if (!xg || !qg) continue;
            for (int64_t j = 0; j < G; ++j) {
                const uint16_t* src = W + n * K + j * g;
                for (int64_t i = 0; i < g; ++i) xg[i] = oracle_bf16_to_f32(src[i]);
                uint16_t s_bits;
                int32_t z = 0;
                if (sym) {
                    oracle_group_sym8(xg, g, &s_bits, qg);
                } else {
                    oracle_group_asym8(xg, g, &s_bits, &z, qg);
                }
                scales[n * G + j] = s_bits;
                if (zeros) zeros[n * G + j] = oracle_f32_to_bf16_rn((float)z);
                for (int64_t i = 0; i < g; ++i)
                    codes[n * K + j * g + i] = (uint8_t)((uint32_t)qg[i] & 0xFFu);
            }
        }
        free(xg);
        free(qg);
    }
    return failed;
}

/* x̂[n, k] = bf16_rn((q − z)·s) from 8-bit codes (R8'). */
int oracle_dequantize8(const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                       int64_t N, int64_t K, int64_t g, int32_t sym, uint16_t* W_hat) {
    if (N < 0 || K < 0 || g <= 0 || K % g != 0) return 1;
    const int64_t G = K / g;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int32_t q = code8_of(codes, n * K + k, sym);
            int64_t j = k / g;
            float s = oracle_bf16_to_f32(scales[n * G + j]);
            int32_t z = sym ? 0 : (int32_t)oracle_bf16_to_f32(zeros[n * G + j]);
            float prod = (float)(q - z) * s;          /* exact: ≤ 8-bit integer × 8-bit significand */
            W_hat[n * K + k] = oracle_f32_to_bf16_rn(prod);
        }
    }
    return 0;
}

/* Y64 at listed (m, n) positions from 8-bit codes, dequantizing row n on the fly. */
int oracle_gemm_w8a16_sampled(const uint16_t* X, int64_t M, int64_t K, const uint8_t* codes,
                              const uint16_t* scales, const uint16_t* zeros, int64_t N,
                              int64_t g, int32_t sym, const int64_t* ms, const int64_t* ns,
                              int64_t count, double* out) {
    if (g <= 0 || K % g != 0) return 1;
    const int64_t G = K / g;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0;
        if (m < 0 || m >= M || n < 0 || n >= N) {
            out[i] = NAN;
            continue;
        }
        for (int64_t k = 0; k < K; ++k) {
            int32_t q = code8_of(codes, n * K + k, sym);
            int64_t j = k / g;
            float s = oracle_bf16_to_f32(scales[n * G + j]);
            int32_t z = sym ? 0 : (int32_t)oracle_bf16_to_f32(zeros[n * G + j]);
            uint16_t w = oracle_f32_to_bf16_rn((float)(q - z) * s);
            acc += (double)oracle_bf16_to_f32(X[m * K + k]) * (double)oracle_bf16_to_f32(w);
        }
        out[i] = acc;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Per-input-channel activation scale: the X/s half of the equivalent
 * per-channel scaling [P2] §三 describes, (X/s)·(s·W) = X·W, with the vector
 * a = 1/s supplied by the caller.  Reading R15: the scaled activation is
 * x' = bf16_rn(x·a) — the product of two bf16 values has at most 16
 * significant bits, so it is exact in binary32 and is rounded once, as if the
 * caller had scaled X in bf16 before the GEMM.
 * ------------------------------------------------------------------------- */
void oracle_scale_activations(const uint16_t* X, int64_t M, int64_t K, const uint16_t* a,
                              uint16_t* Xs) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            float prod = oracle_bf16_to_f32(X[m * K + k]) * oracle_bf16_to_f32(a[k]);
            Xs[m * K + k] = oracle_f32_to_bf16_rn(prod);
        }
    }
}

/* ---------------------------------------------------------------------------
 * W8A8: weights and activations both INT8, for the INT8 tensor cores
 * ("Quantization & Acceleration: 解释 W8A8 与 W4A16 的差异与取舍", 数学机理 (1):
 * both quantized to INT8, activations dynamic and quantized per token;
 * "大模型推理中 Weight-only、W8A8 和 FP8 量化有什么区别？如何选型？", §三: an integer
 * matrix multiply on both 8-bit sides).  Weights: the symmetric 8-bit quantizer
 * above with one group per row (g = K, per output channel).  Activations:
 * symmetric absmax per token (row of X), [P3] §二 with b = 8.
 * Readings: R16 the activation scale s_x = max|x| / 127 stays in binary32
 * (computed per call, never stored in a 16-bit format), q = round(x / s_x) with
 * the binary32 quotient, half to even, clamped to [−128, 127] like the weight
 * codes (never binding: |x| / s_x ≤ 127 up to one rounding); an all-zero row has
 * s_x = 0 and q = 0.  R17 the product is Y = s_x[m]·s_w[n]·Σ_k q_x[m,k]·q_w[n,k]
 * with the integer sum exact (as the INT8 tensor cores accumulate in int32).
 * ------------------------------------------------------------------------- */
void oracle_quantize_act8(const uint16_t* X, int64_t M, int64_t K, int8_t* q, float* s) {
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(oracle_bf16_to_f32(X[m * K + k]));
            if (a > amax) amax = a;
        }
        float sc = amax / 127.0f;
        s[m] = sc;
        for (int64_t k = 0; k < K; ++k) {
            int32_t c = 0;
            if (sc != 0.0f) {
                float r = rintf(oracle_bf16_to_f32(X[m * K + k]) / sc);
                if (r < -128.0f) r = -128.0f;
                if (r > 127.0f) r = 127.0f;
                c = (int32_t)r;
            }
            q[m * K + k] = (int8_t)c;
        }
    }
}

/* Y64[m, n] = s_x[m] · s_w[n] · Σ_k q_x[m, k]·q_w[n, k]: the integer sum exactly
 * (int64), then the two scales and the sum multiplied in binary64.  Weight codes
 * are int8 bytes [N, K] and their scales bf16 [N] (one per output channel). */
void oracle_gemm_w8a8(const int8_t* qx, const float* sx, const int8_t* qw, const uint16_t* sw,
                      int64_t M, int64_t N, int64_t K, double* Y) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k) acc += (int64_t)qx[m * K + k] * (int64_t)qw[n * K + k];
            Y[m * N + n] = (double)sx[m] * (double)oracle_bf16_to_f32(sw[n]) * (double)acc;
        }
    }
}

/* The same value at the listed (m, n) positions only. */
void oracle_gemm_w8a8_sampled(const int8_t* qx, const float* sx, const int8_t* qw, const uint16_t* sw,
                              int64_t K, const int64_t* ms, const int64_t* ns, int64_t count, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        const int64_t m = ms[i], n = ns[i];
        int64_t acc = 0;
        for (int64_t k = 0; k < K; ++k) acc += (int64_t)qx[m * K + k] * (int64_t)qw[n * K + k];
        out[i] = (double)sx[m] * (double)oracle_bf16_to_f32(sw[n]) * (double)acc;
    }
}

/* Elementwise bf16_rn of a binary32 array. */
void oracle_f32_array_to_bf16(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16_rn(x[i]);
}

/* Elementwise bf16_rn of a binary64 array (the comparison target). */
void oracle_round_to_bf16(const double* y, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16_rn(y[i]);
}

/* Number of OpenMP threads the parallel loops above use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
int oracle_num_threads(void) { return 1; }
#endif
