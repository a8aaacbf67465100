/*
 * w4_oracle.c -- plain, slow, obviously-correct CPU oracle for the W4A16 path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its
 * Python binding) may link, import or call this file.  It shares no code, header,
 * table or constant generator with the CUDA kernels; the two meet only through the
 * seeded synthetic inputs.  It is compiled with -ffp-contract=off and without
 * -ffast-math so every float operation below is one IEEE-754 binary32 (or binary64)
 * operation with round-to-nearest-even, in the order written.
 *
 * Sources (page title, section):
 *   [AWQ]  "Quantization Paradigms for Edge Inference: AWQ, GPTQ, and FP8 Matrix Cores",
 *          sec. 3 "The Math Behind Activation-Aware Protection (AWQ)", eq. 1:
 *          W' = W diag(s), X' = diag(s)^-1 X.
 *   [GRP]  "The Ultimate Guide to Quantized LLMs: GPTQ" (refer.kumon.ca), section
 *          "Understanding Quantized Model Compression": calibration fixes per-group
 *          scaling factors and zero points that map high-precision values into a small
 *          integer range.
 *   [RTN]  edgesiliconlab.com article on AWQ vs GPTQ, section "What Is the Core
 *          Difference Between AWQ and GPTQ Quantization?": round-to-nearest into 4-bit
 *          integers; section "Quantization on Non-NVIDIA Silicon": asymmetric affine and
 *          group-wise linear quantization.
 *   [PACK] same article, section "Kernel Execution: Marlin vs. ExLlamaV2 INT4 GEMM
 *          Micro-Architecture", item 3: two 4-bit weights share one byte and are
 *          recovered with shift and AND.
 *   [FP4]  "Production Quantization: AWQ, GPTQ, GGUF K-quants, FP8, MXFP4/NVFP4",
 *          section "MXFP4 / NVFP4" and glossary: block-scaled 4-bit floating point (the
 *          last section of this file; its format readings are stated there).
 *
 * Readings where the pages are silent:
 *   - W is [N,K] row-major (out x in); Y = X' * What^T is [M,N].
 *   - group of channel k: k / group_size, or g_idx[k] when a g_idx array is given.
 *   - asymmetric: sc = fp16(max((max-min)/15, 2^-14)), z = clamp(rint(-min/sc),0,15);
 *     symmetric:  sc = fp16(max(absmax/7, 2^-14)),     z = 8 (not stored).
 *   - quantisation uses the fp16-rounded scale; q = clamp(rint(W'/sc) + z, 0, 15),
 *     rint = round-half-to-even, '/' = IEEE division, clamp taken in float.
 *   - zero points are stored as fp16 values of the integer z.
 *   - canonical packing: word i of row n holds q[n][8i+j] in bits 4j..4j+3.
 *   - device packing: the tile layout stated above oracle_pack_device().
 *   - the reference product is accumulated in fp32 in ascending k (products rounded
 *     to fp32, then added); an fp64 companion exists as a self-check.
 *
 * Parity pins: every function here is pinned by the CPU tests in tests/test_oracle_*.py
 * against closed forms, brute force, library routines or hand-worked values.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if defined(__FAST_MATH__)
#error "the oracle must not be built with -ffast-math"
#endif

/* ------------------------------------------------------------------ */
/* IEEE-754 conversions, written from the format definitions.          */
/* ------------------------------------------------------------------ */

/* round a non-negative, exactly-representable double to the nearest integer,
   ties to even */
static double rne_nonneg(double n) {
    double fl = floor(n);
    double d = n - fl; /* exact */
    if (d > 0.5) return fl + 1.0;
    if (d < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
float oracle_f16_to_f32(uint16_t h) {
    uint32_t sign = (h >> 15) & 1u, e = (h >> 10) & 0x1Fu, m = h & 0x3FFu;
    float v;
    if (e == 0) v = (float)ldexp((double)m, -24);            /* zero / subnormal */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = (float)ldexp((double)(m | 0x400u), (int)e - 25); /* 1.m * 2^(e-15) */
    return sign ? -v : v;
}

uint16_t oracle_f32_to_f16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    if ((x & 0x7F800000u) == 0x7F800000u) return sign | ((x & 0x007FFFFFu) ? 0x7E00u : 0x7C00u);
    double a = fabs((double)f);
    if (a == 0.0) return sign;
    /* largest finite is 65504 = 2047 * 2^5; the midpoint to 2^16 rounds to even (up) */
    if (a >= 65520.0) return sign | 0x7C00u;
    int e2;
    frexp(a, &e2);        /* a = m * 2^e2, 0.5 <= m < 1 */
    int E = e2 - 1;       /* floor(log2 a) */
    if (E < -14) E = -14; /* subnormals share the quantum of the lowest normal binade */
    double quantum = ldexp(1.0, E - 10);
    double r = rne_nonneg(a / quantum); /* a / quantum is exact */
    uint32_t bits;
    if (E == -14) bits = (uint32_t)r;   /* subnormal, or lowest binade (carry is fine) */
    else bits = ((uint32_t)(E + 15) << 10) + ((uint32_t)r - 1024u); /* r in [1024,2048] */
    return (uint16_t)(sign | bits);
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. */
float oracle_bf16_to_f32(uint16_t h) {
    uint32_t x = (uint32_t)h << 16;
    float f;
    memcpy(&f, &x, 4);
    return f;
}

uint16_t oracle_f32_to_bf16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    if ((x & 0x7F800000u) == 0x7F800000u) return sign | ((x & 0x007FFFFFu) ? 0x7FC0u : 0x7F80u);
    double a = fabs((double)f);
    if (a == 0.0) return sign;
    /* largest finite is 255 * 2^120; the midpoint to 2^128 is 511 * 2^119 */
    if (a >= ldexp(511.0, 119)) return sign | 0x7F80u;
    int e2;
    frexp(a, &e2);
    int E = e2 - 1;
    if (E < -126) E = -126;
    double quantum = ldexp(1.0, E - 7);
    double r = rne_nonneg(a / quantum);
    uint32_t bits;
    if (E == -126) bits = (uint32_t)r;
    else bits = ((uint32_t)(E + 127) << 7) + ((uint32_t)r - 128u);
    return (uint16_t)(sign | bits);
}

/* element of a 16-bit activation / weight array as fp32 */
static float load16(const uint16_t* p, int64_t i, int is_bf16) {
    return is_bf16 ? oracle_bf16_to_f32(p[i]) : oracle_f16_to_f32(p[i]);
}

/* bulk helpers so the tests can pin the converters over whole arrays */
void oracle_f16_to_f32_array(const uint16_t* h, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f32(h[i]);
}
void oracle_f32_to_f16_array(const float* f, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16(f[i]);
}
void oracle_bf16_to_f32_array(const uint16_t* h, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_f32(h[i]);
}
void oracle_f32_to_bf16_array(const float* f, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(f[i]);
}

/* ------------------------------------------------------------------ */
/* [AWQ] eq. 1, weight side: W'[n,k] = fp32(W[n,k]) * s[k], one fp32    */
/* rounding; W' = fp32(W) when s is NULL.                               */
/* ------------------------------------------------------------------ */
void oracle_awq_scale_weights(const uint16_t* W, int w_is_bf16, int64_t N, int64_t K,
                              const float* s, float* Wp) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float w = load16(W, n * K + k, w_is_bf16);
            Wp[n * K + k] = s ? w * s[k] : w;
        }
}

/* [AWQ] eq. 1, activation side: X'[m,k] = fp32(X[m,k]) * s_inv[k]. */
void oracle_awq_scale_acts(const uint16_t* X, int x_is_bf16, int64_t M, int64_t K,
                           const float* s_inv, float* Xp) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            float x = load16(X, m * K + k, x_is_bf16);
            Xp[m * K + k] = s_inv ? x * s_inv[k] : x;
        }
}

static int64_t group_of(int64_t k, int32_t group_size, const int32_t* g_idx) {
    return g_idx ? (int64_t)g_idx[k] : k / group_size;
}

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ------------------------------------------------------------------ */
/* [GRP]+[RTN]: group-wise round-to-nearest INT4 of the scaled weights. */
/* Wp fp32 [N,K]; outputs q uint8 [N,K] (codes 0..15), scales fp16 bits */
/* [G,N], zeros fp16 bits [G,N] (asymmetric only; may be NULL when       */
/* symmetric).  Returns 0, or -1 on bad arguments.                       */
/* ------------------------------------------------------------------ */
int oracle_quantize(const float* Wp, int64_t N, int64_t K, int32_t group_size, int symmetric,
                    const int32_t* g_idx, uint8_t* q, uint16_t* scales, uint16_t* zeros) {
    if (N <= 0 || K <= 0 || group_size <= 0 || K % group_size != 0) return -1;
    int64_t G = K / group_size;
    if (g_idx)
        for (int64_t k = 0; k < K; ++k)
            if (g_idx[k] < 0 || g_idx[k] >= G) return -1;
    float* mn = (float*)malloc(sizeof(float) * (size_t)G);
    float* mx = (float*)malloc(sizeof(float) * (size_t)G);
    float* am = (float*)malloc(sizeof(float) * (size_t)G);
    float* sc = (float*)malloc(sizeof(float) * (size_t)G);
    float* zf = (float*)malloc(sizeof(float) * (size_t)G);
    if (!mn || !mx || !am || !sc || !zf) {
        free(mn); free(mx); free(am); free(sc); free(zf);
        return -1;
    }
    const float min_scale = 0x1p-14f; /* smallest normal binary16 */
    for (int64_t n = 0; n < N; ++n) {
        const float* row = Wp + n * K;
        for (int64_t g = 0; g < G; ++g) { mn[g] = INFINITY; mx[g] = -INFINITY; am[g] = 0.0f; }
        /* step 1: range of every group */
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = group_of(k, group_size, g_idx);
            float v = row[k];
            if (v < mn[g]) mn[g] = v;
            if (v > mx[g]) mx[g] = v;
            if (fabsf(v) > am[g]) am[g] = fabsf(v);
        }
        /* step 2: scale (rounded to fp16) and integer zero point */
        for (int64_t g = 0; g < G; ++g) {
            float s_f = symmetric ? am[g] / 7.0f : (mx[g] - mn[g]) / 15.0f;
            if (s_f < min_scale) s_f = min_scale;
            uint16_t s16 = oracle_f32_to_f16(s_f);
            sc[g] = oracle_f16_to_f32(s16);
            scales[g * N + n] = s16;
            if (symmetric) {
                zf[g] = 8.0f;
            } else {
                /* z is an integer in [0,15]: rint(-(+0)) = -0 must be stored as +0 */
                int zi = (int)clampf(rintf(-mn[g] / sc[g]), 0.0f, 15.0f);
                zf[g] = (float)zi;
                if (zeros) zeros[g * N + n] = oracle_f32_to_f16(zf[g]);
            }
        }
        /* step 3: round to nearest (ties to even), shift by the zero point, clamp */
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = group_of(k, group_size, g_idx);
            float t = rintf(row[k] / sc[g]);
            q[n * K + k] = (uint8_t)clampf(t + zf[g], 0.0f, 15.0f);
        }
    }
    free(mn); free(mx); free(am); free(sc); free(zf);
    return 0;
}

/* ------------------------------------------------------------------ */
/* [PACK] canonical packing: uint32 [N, K/8]; nibble j of word i of row  */
/* n is q[n][8i+j] (bits 4j..4j+3).                                      */
/* ------------------------------------------------------------------ */
void oracle_pack_canonical(const uint8_t* q, int64_t N, int64_t K, uint32_t* qc) {
    int64_t W = K / 8;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t i = 0; i < W; ++i) {
            uint32_t w = 0;
            for (int j = 0; j < 8; ++j) w |= (uint32_t)(q[n * K + 8 * i + j] & 0xF) << (4 * j);
            qc[n * W + i] = w;
        }
}

void oracle_unpack_canonical(const uint32_t* qc, int64_t N, int64_t K, uint8_t* q) {
    int64_t W = K / 8;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t i = 0; i < W; ++i)
            for (int j = 0; j < 8; ++j)
                q[n * K + 8 * i + j] = (uint8_t)((qc[n * W + i] >> (4 * j)) & 0xF);
}

/* ------------------------------------------------------------------ */
/* Device packing (the library's own layout; N % 16 == 0, K % 64 == 0).  */
/* The weight matrix is cut into atoms of 16 rows x 64 columns.  Eight   */
/* consecutive row tiles form a band of 128 rows (the last band holds    */
/* Tb = min(8, N/16 - 8b) tiles).  Band b starts at atom 8*(K/64)*b and  */
/* inside it atom (tile tt of the band, column block a) is atom           */
/* a*Tb + tt; atom i occupies words 128*i .. 128*i+127.  Inside an atom,  */
/* word 4*L + j (L = 0..31, j = 0..3) holds, for r0 = 16t + L/4 (t the    */
/* tile's row index), r1 = r0 + 8, kb = 64a + 16j, c = 2*(L%4), the codes */
/*   nibble 0: q[r0][kb+c]    nibble 4: q[r0][kb+c+1]                     */
/*   nibble 1: q[r1][kb+c]    nibble 5: q[r1][kb+c+1]                     */
/*   nibble 2: q[r0][kb+c+8]  nibble 6: q[r0][kb+c+9]                     */
/*   nibble 3: q[r1][kb+c+8]  nibble 7: q[r1][kb+c+9]                     */
/* with nibble i in bits 4i..4i+3.                                        */
/* ------------------------------------------------------------------ */
static void device_slot(int64_t N, int64_t K, int64_t word, int nib, int64_t* n, int64_t* k) {
    int64_t KA = K / 64, T = N / 16;
    int64_t atom = word / 128, inw = word % 128;
    int64_t b = atom / (8 * KA), in_band = atom % (8 * KA);
    int64_t Tb = (T - 8 * b) < 8 ? (T - 8 * b) : 8;
    int64_t a = in_band / Tb, t = 8 * b + in_band % Tb;
    int64_t L = inw / 4, j = inw % 4;
    int64_t r0 = 16 * t + L / 4, c = 2 * (L % 4), kb = 64 * a + 16 * j;
    static const int row_hi[8] = {0, 1, 0, 1, 0, 1, 0, 1};
    static const int col_off[8] = {0, 0, 8, 8, 1, 1, 9, 9};
    *n = r0 + 8 * row_hi[nib];
    *k = kb + c + col_off[nib];
}

int oracle_pack_device(const uint8_t* q, int64_t N, int64_t K, uint32_t* qd) {
    if (N % 16 || K % 64) return -1;
    int64_t words = N * K / 8;
    for (int64_t w = 0; w < words; ++w) {
        uint32_t v = 0;
        for (int i = 0; i < 8; ++i) {
            int64_t n, k;
            device_slot(N, K, w, i, &n, &k);
            v |= (uint32_t)(q[n * K + k] & 0xF) << (4 * i);
        }
        qd[w] = v;
    }
    return 0;
}

int oracle_unpack_device(const uint32_t* qd, int64_t N, int64_t K, uint8_t* q) {
    if (N % 16 || K % 64) return -1;
    int64_t words = N * K / 8;
    for (int64_t w = 0; w < words; ++w)
        for (int i = 0; i < 8; ++i) {
            int64_t n, k;
            device_slot(N, K, w, i, &n, &k);
            q[n * K + k] = (uint8_t)((qd[w] >> (4 * i)) & 0xF);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Dequantisation: What[n,k] = (q - z) * sc, exact in fp32 (|q - z| has  */
/* at most 4 bits, sc an 11-bit significand).  zeros == NULL means the   */
/* symmetric format with z = 8.                                          */
/* ------------------------------------------------------------------ */
void oracle_dequant(const uint8_t* q, const uint16_t* scales, const uint16_t* zeros,
                    const int32_t* g_idx, int32_t group_size, int64_t N, int64_t K, float* What) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = group_of(k, group_size, g_idx);
            float sc = oracle_f16_to_f32(scales[g * N + n]);
            float z = zeros ? oracle_f16_to_f32(zeros[g * N + n]) : 8.0f;
            What[n * K + k] = ((float)q[n * K + k] - z) * sc;
        }
}

/* ------------------------------------------------------------------ */
/* Reference product Y[m,n] = sum_k X'[m,k] * What[n,k].                 */
/* rows: optional list of nrows row indices of X' to evaluate (NULL =    */
/* all M rows); Y has one row per evaluated row.                         */
/* ------------------------------------------------------------------ */
void oracle_gemm_f32(const float* Xp, const float* What, int64_t M, int64_t N, int64_t K,
                     const int64_t* rows, int64_t nrows, float* Y) {
    int64_t R = rows ? nrows : M;
    for (int64_t i = 0; i < R; ++i) {
        const float* x = Xp + (rows ? rows[i] : i) * K;
        for (int64_t n = 0; n < N; ++n) {
            const float* w = What + n * K;
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float p = x[k] * w[k];
                acc = acc + p;
            }
            Y[i * N + n] = acc;
        }
    }
}

void oracle_gemm_f64(const float* Xp, const float* What, int64_t M, int64_t N, int64_t K,
                     const int64_t* rows, int64_t nrows, double* Y) {
    int64_t R = rows ? nrows : M;
    for (int64_t i = 0; i < R; ++i) {
        const float* x = Xp + (rows ? rows[i] : i) * K;
        for (int64_t n = 0; n < N; ++n) {
            const float* w = What + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += (double)x[k] * (double)w[k];
            Y[i * N + n] = acc;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Block-scaled 4-bit floating point (NVFP4, MXFP4).                   */
/* ------------------------------------------------------------------ */
/* "Production Quantization: AWQ, GPTQ, GGUF K-quants, FP8, MXFP4/NVFP4", section
 * "MXFP4 / NVFP4" and its glossary: microscaling 4-bit floating point in which every
 * block of weights carries its own scale factor, run by Blackwell's tensor cores.  The
 * pages fix nothing further; the encodings below are the formats' published
 * definitions, taken as readings:
 *   element  E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 *            0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinity or NaN.
 *   NVFP4    blocks of 16 consecutive k, an E4M3 block scale (bias 7, no infinity,
 *            largest finite 448) and one fp32 scale for the whole tensor:
 *              gs = amax / (6 * 448)  (1 for an all-zero tensor),
 *              sb = E4M3(blockmax / 6 / gs),   q = E2M1(w / (dec(sb) * gs)).
 *   MXFP4    blocks of 32, a power-of-two scale 2^e stored as the byte e + 127 (E8M0),
 *              e = floor(log2(blockmax)) - 2   (2 = the largest E2M1 exponent),
 *              q = E2M1(w / 2^e).
 * Every encoding rounds to the nearest representable value, ties to the even
 * mantissa, and saturates finite values beyond the largest magnitude.  The search is
 * exhaustive over the codes, which is the definition of round-to-nearest. */

float oracle_e2m1_to_f32(uint8_t c) {
    const int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    const float mag = e == 0 ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
    return s ? -mag : mag;
}

uint8_t oracle_f32_to_e2m1(float x) {
    const double a = fabs((double)x);
    uint8_t best = 0;
    double bd = INFINITY;
    for (uint8_t c = 0; c < 8; ++c) {
        const double d = fabs(a - (double)oracle_e2m1_to_f32(c));
        if (d < bd || (d == bd && (c & 1) == 0)) {
            bd = d;
            best = c;
        }
    }
    return (uint8_t)((signbit(x) ? 8 : 0) | best);
}

float oracle_e4m3_to_f32(uint8_t b) {
    const int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    float mag;
    if (e == 15 && m == 7) mag = NAN;
    else if (e == 0) mag = ldexpf((float)m, -9);               /* (m/8) 2^-6 */
    else mag = ldexpf((float)(8 + m), e - 10);                 /* (1 + m/8) 2^(e-7) */
    return s ? -mag : mag;
}

uint8_t oracle_f32_to_e4m3(float x) {
    const double a = fabs((double)x);
    uint8_t best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 127; ++c) {                           /* 127 = NaN */
        const double d = fabs(a - (double)oracle_e4m3_to_f32((uint8_t)c));
        if (d < bd || (d == bd && (c & 1) == 0)) {
            bd = d;
            best = (uint8_t)c;
        }
    }
    return (uint8_t)((signbit(x) ? 0x80 : 0) | best);
}

/* NVFP4 of A [R,K] (fp16/bf16 bits), K % 16 == 0: codes [R,K] one E2M1 code per byte,
   block scales [R,K/16] E4M3 bytes, *gs the tensor scale.  Returns 0, -1 on bad K. */
int oracle_nvfp4_quantize(const uint16_t* A, int is_bf16, int64_t R, int64_t K,
                          uint8_t* codes, uint8_t* bscale, float* gs) {
    if (K % 16 != 0) return -1;
    float amax = 0.0f;
    for (int64_t i = 0; i < R * K; ++i) amax = fmaxf(amax, fabsf(load16(A, i, is_bf16)));
    const float g = amax > 0.0f ? amax / (6.0f * 448.0f) : 1.0f;
    *gs = g;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t b = 0; b < K / 16; ++b) {
            float bmax = 0.0f;
            for (int64_t k = 16 * b; k < 16 * b + 16; ++k) bmax = fmaxf(bmax, fabsf(load16(A, r * K + k, is_bf16)));
            const uint8_t sb = oracle_f32_to_e4m3(bmax / 6.0f / g);
            bscale[r * (K / 16) + b] = sb;
            const float sd = oracle_e4m3_to_f32(sb) * g;
            for (int64_t k = 16 * b; k < 16 * b + 16; ++k) {
                const float w = load16(A, r * K + k, is_bf16);
                codes[r * K + k] = sd > 0.0f ? oracle_f32_to_e2m1(w / sd) : 0;
            }
        }
    return 0;
}

/* dequantised NVFP4 values: A^[r,k] = E2M1(code) * (E4M3(sb) * gs), in fp64 (exact:
   the first factor has 2 significant bits, the block scale 4, gs is one fp32). */
void oracle_nvfp4_dequant(const uint8_t* codes, const uint8_t* bscale, float gs, int64_t R, int64_t K,
                          double* out) {
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = (double)oracle_e2m1_to_f32(codes[r * K + k]) *
                             (double)oracle_e4m3_to_f32(bscale[r * (K / 16) + k / 16]) * (double)gs;
}

/* MXFP4 of A [R,K], K % 32 == 0: codes [R,K], scale bytes [R,K/32] (E8M0: 2^(byte-127)). */
int oracle_mxfp4_quantize(const uint16_t* A, int is_bf16, int64_t R, int64_t K, uint8_t* codes,
                          uint8_t* escale) {
    if (K % 32 != 0) return -1;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t b = 0; b < K / 32; ++b) {
            float bmax = 0.0f;
            for (int64_t k = 32 * b; k < 32 * b + 32; ++k) bmax = fmaxf(bmax, fabsf(load16(A, r * K + k, is_bf16)));
            int e = -127;
            if (bmax > 0.0f) {
                int ex;
                (void)frexpf(bmax, &ex);                       /* bmax = f 2^ex, f in [0.5, 1) */
                e = ex - 1 - 2;
                if (e < -127) e = -127;
            }
            escale[r * (K / 32) + b] = (uint8_t)(e + 127);
            for (int64_t k = 32 * b; k < 32 * b + 32; ++k)
                codes[r * K + k] = oracle_f32_to_e2m1(ldexpf(load16(A, r * K + k, is_bf16), -e));
        }
    return 0;
}

void oracle_mxfp4_dequant(const uint8_t* codes, const uint8_t* escale, int64_t R, int64_t K, double* out) {
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = ldexp((double)oracle_e2m1_to_f32(codes[r * K + k]),
                                   (int)escale[r * (K / 32) + k / 32] - 127);
}
