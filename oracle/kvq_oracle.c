/*
 * kvq_oracle.c -- plain, slow, obviously-correct CPU oracle for quantized-KV
 * decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / --impl reference legs of bench.py may load or call this code.
 * It shares nothing (no header, helper, table or constant) with the CUDA
 * library under quantized_kv_cache_22_b200/csrc, and never imports it.
 *
 * What it computes, and where that is stated:
 *
 *  - Symmetric absmax quantisation, 255 levels for INT8 (codes -127..127) and
 *    15 levels for INT4 (codes -7..7), one fp16 scale per group of elements.
 *    TinyLoop docs "KV Cache 模式", table of the five modes (INT8 KV row: two
 *    INT8 vectors plus one FP16 scale per head; INT4 h row: nibble-packed with
 *    per-head FP16 scales, "15 levels" vs "255 levels").  Group-of-32 scales:
 *    KVSplit page, "So sánh hiệu quả tiết kiệm bộ nhớ" (93.5 / 71.5 / 49.5 MB
 *    at 8K tokens are exactly 8.5 and 4.5 bits per element).
 *    The pages fix no rounding rule; the readings taken here are:
 *      s32  = absmax / qmax                 (IEEE fp32 division)
 *      s16  = fp16_rne(s32), +inf saturated to 65504, subnormals kept
 *      code = clamp(rne(x / float(s16)), -qmax, qmax), all zero if s16 == 0
 *      INT4 packing: element 2j in the low nibble, 2j+1 in the high nibble,
 *      4-bit two's complement.
 *  - Decode attention: s_t = tau * q . k^_t, p = softmax(s) over every cached
 *    token, o = sum_t p_t v^_t, all in fp64 (the problem statement on the
 *    mni-ml page, "Cách KV cache tạo ra tốc độ": keep K and V of past tokens,
 *    compute only the new token's).  Query head h reads KV head floor(h / G).
 *  - h-mode (TinyLoop docs, "運作原理"): cache h, rebuild K = W_k h and
 *    V = W_v h at every attention call.  Here h^ is dequantised, rounded to
 *    bf16 (the GEMM operand), K/V = W h^ in fp64 with W bf16, rounded to fp16.
 *  - FP8 e4m3 codes (the mni-ml page's comparison with production stacks:
 *    vLLM and TensorRT-LLM keep FP8 KV caches): same fp16 scales, with 448
 *    (the largest finite e4m3 magnitude) in place of qmax and
 *    code = e4m3_rne(x / s), saturating.  Bit-width code KVQO_E4M3 (228).
 *  - Asymmetric INT8 with a zero-point, and per-tensor INT8 (the mni-ml page,
 *    "Tại sao INT8 mà không mất tốc": scale/zero-point metadata; "Limitations":
 *    symmetric per-tensor scaling).  Asymmetric, per group of elements, the
 *    textbook affine scheme with zero inside the range:
 *      lo = min(0, min x), hi = max(0, max x)
 *      s16 = fp16_rne((hi - lo) / 255), +inf saturated to 65504
 *      z = clamp(rne(-lo / s), 0, 255),  q = clamp(rne(x / s) + z, 0, 255)
 *      x^ = (q - z) * s;  s == 0: z = 0 and q = 0.
 *    q is stored as a uint8, and each group keeps the pair (s16, fp16(z)).
 *    Bit-width code KVQO_ASYM8 (208).  Per-tensor: one caller-given fp16
 *    scale s for a whole tensor, code = clamp(rne(x / s), -127, 127), the
 *    symmetric INT8 codes (x^ = code * s, the per-head dequantisation with
 *    every row's scale equal to s).
 *  - h-mode decode by query absorption: the same attention as the
 *    reconstruction path, regrouped by linearity (qa = W_k^T q, s = qa . h^,
 *    out = W_v sum_t p_t h^_t), in fp64 without the bf16 / fp16 roundings.
 *  - Bytes per token per layer (TinyLoop docs, "記憶體公式" table).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -ffp-contract=off (no fast-math: the
 * quantiser's divisions must be IEEE).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KVQO_E4M3 228   /* bit-width code for FP8 e4m3 codes (8 bits per element) */
#define KVQO_ASYM8 208  /* bit-width code for asymmetric INT8 (uint8 codes, (scale, zero) pairs) */

/* ------------------------------------------------------------------------ */
/* Binary16 / bfloat16 conversions written from the IEEE 754 definitions.    */
/* ------------------------------------------------------------------------ */

/* Round a non-negative integer significand `m` (value m * 2^e2) to the
 * binary16 grid and return the encoded magnitude (no sign).  Used by both the
 * float and double converters.  `m` has `mbits` significant bits at most. */
static uint16_t f16_from_parts(uint64_t m, int e2)
{
    /* value = m * 2^e2, m > 0.  Find the binade: top bit position. */
    int top = 63;
    while (top >= 0 && !((m >> top) & 1u)) top--;
    if (top < 0) return 0;
    int e = top + e2;               /* unbiased exponent of the value        */
    int ulp_exp = (e >= -14) ? e - 10 : -24;  /* binary16 ulp at this value  */
    int shift = ulp_exp - e2;       /* bits of m below the binary16 ulp       */
    uint64_t q;
    if (shift <= 0) {
        q = m << (-shift);          /* exact (only for tiny m)               */
    } else if (shift >= 64) {
        q = 0;                      /* far below half an ulp: rounds to 0    */
        /* m < 2^(top+1) <= 2^64 and half ulp = 2^(shift-1) >= 2^63.  A tie
         * would need m == 2^63 exactly with shift == 64; then q=0 is even. */
    } else {
        q = m >> shift;
        uint64_t rem = m & ((((uint64_t)1) << shift) - 1);
        uint64_t half = ((uint64_t)1) << (shift - 1);
        if (rem > half || (rem == half && (q & 1))) q++;
    }
    /* q is the significand in units of the binary16 ulp. */
    if (e >= -14) {
        if (q >= 2048) {            /* rounding carried into the next binade */
            q >>= 1;
            e += 1;
        }
        if (e > 15) return 0x7c00;  /* overflow to infinity                  */
        return (uint16_t)(((e + 15) << 10) | (q & 0x3ff));
    }
    /* subnormal range: q in units of 2^-24; q == 1024 encodes 2^-14 exactly */
    return (uint16_t)q;
}

uint16_t kvqo_f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u) return sign | 0x7e00;     /* NaN                   */
    if (ax == 0x7f800000u) return sign | 0x7c00;    /* infinity              */
    if (ax == 0) return sign;
    uint32_t be = ax >> 23, fr = ax & 0x7fffffu;
    uint64_t m = be ? (fr | 0x800000u) : fr;
    int e2 = (be ? (int)be : 1) - 127 - 23;
    return sign | f16_from_parts(m, e2);
}

uint16_t kvqo_f64_to_f16(double d)
{
    uint64_t x;
    memcpy(&x, &d, 8);
    uint16_t sign = (uint16_t)((x >> 48) & 0x8000u);
    uint64_t ax = x & 0x7fffffffffffffffull;
    if (ax > 0x7ff0000000000000ull) return sign | 0x7e00;
    if (ax == 0x7ff0000000000000ull) return sign | 0x7c00;
    if (ax == 0) return sign;
    uint64_t be = ax >> 52, fr = ax & 0xfffffffffffffull;
    uint64_t m = be ? (fr | 0x10000000000000ull) : fr;
    int e2 = (be ? (int)be : 1) - 1023 - 52;
    return sign | f16_from_parts(m, e2);
}

float kvqo_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int be = (h >> 10) & 0x1f;
    int fr = h & 0x3ff;
    float v;
    if (be == 0x1f) v = fr ? NAN : INFINITY;
    else if (be == 0) v = ldexpf((float)fr, -24);
    else v = ldexpf((float)(fr | 0x400), be - 25);
    return sign ? -v : v;
}

/* bfloat16: keep the top 16 bits of the binary32 encoding, rounding the
 * dropped 16 bits to nearest, ties to even. */
uint16_t kvqo_f32_to_bf16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    if ((x & 0x7fffffffu) > 0x7f800000u) return (uint16_t)(((x >> 16) & 0x8000u) | 0x7fc0u);
    uint32_t lo = x & 0xffffu, hi = x >> 16;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1;
    return (uint16_t)hi;
}

float kvqo_bf16_to_f32(uint16_t b)
{
    uint32_t x = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &x, 4);
    return f;
}

/* ------------------------------------------------------------------------ */
/* FP8 e4m3 ("fn": 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,  */
/* no infinities; 0x7f / 0xff are NaN; the largest finite magnitude is 448 =  */
/* 1.75 * 2^8, the smallest subnormal 2^-9).                                  */
/* ------------------------------------------------------------------------ */

/* Encode a float, rounding to nearest with ties to even; magnitudes that would
 * round above 448 saturate to 448 (the KV-cache use never wants NaN). */
uint8_t kvqo_f32_to_e4m3(float f)
{
    const uint8_t sign = signbit(f) ? 0x80 : 0x00;
    if (isnan(f)) return (uint8_t)(sign | 0x7f);
    const float a = fabsf(f);
    if (a == 0.0f) return sign;
    if (a < 0.015625f) {
        /* below the smallest normal 2^-6: multiples of 2^-9 (a code of 8 is 2^-6,
         * which is also the encoding of the smallest normal) */
        const float m = nearbyintf(a * 512.0f);
        return (uint8_t)(sign | (uint8_t)m);
    }
    int ex = 0;
    (void)frexpf(a, &ex);           /* a = fr * 2^ex, fr in [0.5, 1) */
    int e = ex - 1;                 /* a in [2^e, 2^(e+1)) */
    if (e > 8) return (uint8_t)(sign | 0x7e);
    float m = nearbyintf(ldexpf(a, 3 - e));  /* 8 .. 16: significand in eighths */
    if (m == 16.0f) {
        m = 8.0f;
        e += 1;
    }
    const int code = ((e + 7) << 3) | ((int)m - 8);
    if (code > 0x7e) return (uint8_t)(sign | 0x7e);
    return (uint8_t)(sign | code);
}

float kvqo_e4m3_to_f32(uint8_t c)
{
    const float sgn = (c & 0x80) ? -1.0f : 1.0f;
    const int e = (c >> 3) & 0xf, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) return sgn * ldexpf((float)m, -9);
    return sgn * ldexpf((float)(8 + m), e - 10);
}

/* ------------------------------------------------------------------------ */
/* Quantiser                                                                 */
/* ------------------------------------------------------------------------ */

static int qmax_of(int bits) { return bits == 8 ? 127 : 7; }

/* FP8 codes: scale s = fp16(absmax / 448), code = e4m3(x / s) (saturating). */
static void quantize_group_e4m3(const float *x, int n, uint8_t *codes, uint16_t *scale_out)
{
    float a = 0.0f;
    for (int i = 0; i < n; i++) {
        float v = fabsf(x[i]);
        if (v > a) a = v;
    }
    float s32 = a / 448.0f;
    uint16_t s16 = kvqo_f32_to_f16(s32);
    if ((s16 & 0x7fffu) == 0x7c00u) s16 = (uint16_t)((s16 & 0x8000u) | 0x7bffu);
    float s = kvqo_f16_to_f32(s16);
    for (int i = 0; i < n; i++) codes[i] = (s == 0.0f) ? 0 : kvqo_f32_to_e4m3(x[i] / s);
    *scale_out = s16;
}

/* Asymmetric INT8: lo = min(0, min x), hi = max(0, max x), s = fp16((hi-lo)/255),
 * z = clamp(rne(-lo/s), 0, 255), q = clamp(rne(x/s) + z, 0, 255). */
static void quantize_group_asym8(const float *x, int n, uint8_t *codes, uint16_t *scale_out,
                                 uint16_t *zero_out)
{
    float lo = 0.0f, hi = 0.0f;
    for (int i = 0; i < n; i++) {
        if (x[i] < lo) lo = x[i];
        if (x[i] > hi) hi = x[i];
    }
    float s32 = (hi - lo) / 255.0f;
    uint16_t s16 = kvqo_f32_to_f16(s32);
    if ((s16 & 0x7fffu) == 0x7c00u) s16 = (uint16_t)((s16 & 0x8000u) | 0x7bffu);
    float s = kvqo_f16_to_f32(s16);
    int z = 0;
    if (s != 0.0f) {
        float zr = nearbyintf(-lo / s);
        if (zr < 0.0f) zr = 0.0f;
        if (zr > 255.0f) zr = 255.0f;
        z = (int)zr;
    }
    for (int i = 0; i < n; i++) {
        if (s == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float r = nearbyintf(x[i] / s) + (float)z;
        if (r < 0.0f) r = 0.0f;
        if (r > 255.0f) r = 255.0f;
        codes[i] = (uint8_t)(int)r;
    }
    *scale_out = s16;
    *zero_out = kvqo_f32_to_f16((float)z);
}

/* Per-tensor INT8 with a given fp16 scale s16: code = clamp(rne(x / s), -127, 127),
 * all codes 0 when s == 0.  n_rows x dim floats, one byte per element. */
int kvqo_quantize_rows_tensor(const float *x, int64_t n_rows, int dim, uint16_t s16,
                              uint8_t *codes)
{
    const float s = kvqo_f16_to_f32(s16);
    if (!(s >= 0.0f) || isinf(s)) return -1;
    for (int64_t i = 0; i < n_rows * (int64_t)dim; i++) {
        if (s == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float r = nearbyintf(x[i] / s);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        codes[i] = (uint8_t)(int8_t)(int)r;
    }
    return 0;
}

/* Quantise one group of n floats.  codes[i] receives the signed code. */
static void quantize_group(const float *x, int n, int bits, int *codes, uint16_t *scale_out)
{
    const int qmax = qmax_of(bits);
    float a = 0.0f;
    for (int i = 0; i < n; i++) {
        float v = fabsf(x[i]);
        if (v > a) a = v;
    }
    float s32 = a / (float)qmax;
    uint16_t s16 = kvqo_f32_to_f16(s32);
    if ((s16 & 0x7fffu) == 0x7c00u) s16 = (uint16_t)((s16 & 0x8000u) | 0x7bffu);
    float s = kvqo_f16_to_f32(s16);
    for (int i = 0; i < n; i++) {
        if (s == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float r = nearbyintf(x[i] / s);
        if (r > (float)qmax) r = (float)qmax;
        if (r < (float)-qmax) r = (float)-qmax;
        codes[i] = (int)r;
    }
    *scale_out = s16;
}

/* Quantise n_rows rows of `dim` floats with groups of `group` elements at
 * `bits` (4 or 8).  Output codes are row-major, dim*bits/8 bytes per row;
 * scales are row-major, dim/group fp16 values per row. */
int kvqo_quantize_rows(const float *x, int64_t n_rows, int dim, int group, int bits,
                       uint8_t *codes, uint16_t *scales)
{
    if (bits == KVQO_ASYM8) {
        /* scales: [n_rows][dim/group][2] = (s16, fp16(z)) per group */
        if (group <= 0 || dim % group != 0) return -1;
        const int ng = dim / group;
        for (int64_t r = 0; r < n_rows; r++)
            for (int g = 0; g < ng; g++)
                quantize_group_asym8(x + r * (int64_t)dim + g * group, group,
                                     codes + r * (int64_t)dim + g * group,
                                     &scales[(r * ng + g) * 2], &scales[(r * ng + g) * 2 + 1]);
        return 0;
    }
    if (bits == KVQO_E4M3) {
        if (group <= 0 || dim % group != 0) return -1;
        const int ng = dim / group;
        for (int64_t r = 0; r < n_rows; r++)
            for (int g = 0; g < ng; g++)
                quantize_group_e4m3(x + r * (int64_t)dim + g * group, group,
                                    codes + r * (int64_t)dim + g * group, &scales[r * ng + g]);
        return 0;
    }
    if (bits != 4 && bits != 8) return -1;
    if (group <= 0 || dim % group != 0) return -1;
    if (bits == 4 && (group % 2 != 0)) return -1;
    int *tmp = (int *)malloc(sizeof(int) * (size_t)dim);
    if (!tmp) return -2;
    const int ng = dim / group;
    const int row_bytes = dim * bits / 8;
    for (int64_t r = 0; r < n_rows; r++) {
        const float *xr = x + r * (int64_t)dim;
        for (int g = 0; g < ng; g++)
            quantize_group(xr + g * group, group, bits, tmp + g * group, &scales[r * ng + g]);
        uint8_t *cr = codes + r * (int64_t)row_bytes;
        if (bits == 8) {
            for (int i = 0; i < dim; i++) cr[i] = (uint8_t)(int8_t)tmp[i];
        } else {
            for (int j = 0; j < dim / 2; j++) {
                uint8_t lo = (uint8_t)(tmp[2 * j] & 0xf);
                uint8_t hi = (uint8_t)(tmp[2 * j + 1] & 0xf);
                cr[j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    free(tmp);
    return 0;
}

/* Read back signed code i of a packed row. */
static int code_at(const uint8_t *row, int i, int bits)
{
    if (bits == 8) return (int)(int8_t)row[i];
    int nib = (row[i >> 1] >> ((i & 1) * 4)) & 0xf;
    return nib >= 8 ? nib - 16 : nib;
}

/* Dequantise rows: x^_i = code_i * float(s16) (exact in fp32 and fp64).
 * bits == 16 means the row already holds fp16 values (scales ignored). */
int kvqo_dequantize_rows(const uint8_t *codes, const uint16_t *scales, int64_t n_rows, int dim,
                         int group, int bits, double *out)
{
    if (bits == 16) {
        const uint16_t *h = (const uint16_t *)codes;
        for (int64_t i = 0; i < n_rows * (int64_t)dim; i++) out[i] = (double)kvqo_f16_to_f32(h[i]);
        return 0;
    }
    if (bits == KVQO_ASYM8) {
        if (group <= 0 || dim % group != 0) return -1;
        const int ng = dim / group;
        for (int64_t r = 0; r < n_rows; r++)
            for (int i = 0; i < dim; i++) {
                const int64_t gi = (r * ng + i / group) * 2;
                const double sc = (double)kvqo_f16_to_f32(scales[gi]);
                const double z = (double)kvqo_f16_to_f32(scales[gi + 1]);
                out[r * dim + i] = ((double)codes[r * (int64_t)dim + i] - z) * sc;
            }
        return 0;
    }
    if (bits == KVQO_E4M3) {
        if (group <= 0 || dim % group != 0) return -1;
        const int ng = dim / group;
        for (int64_t r = 0; r < n_rows; r++)
            for (int i = 0; i < dim; i++)
                out[r * dim + i] = (double)kvqo_e4m3_to_f32(codes[r * (int64_t)dim + i]) *
                                   (double)kvqo_f16_to_f32(scales[r * ng + i / group]);
        return 0;
    }
    if (bits != 4 && bits != 8) return -1;
    if (group <= 0 || dim % group != 0) return -1;
    const int ng = dim / group;
    const int row_bytes = dim * bits / 8;
    for (int64_t r = 0; r < n_rows; r++) {
        const uint8_t *cr = codes + r * (int64_t)row_bytes;
        for (int i = 0; i < dim; i++) {
            float s = kvqo_f16_to_f32(scales[r * ng + i / group]);
            out[r * dim + i] = (double)code_at(cr, i, bits) * (double)s;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                 */
/* ------------------------------------------------------------------------ */

/* One query vector against L cached (dequantised) keys and values, fp64.
 * No mask: a decode query sees every cached token.  L == 0 gives zeros. */
int kvqo_attend(const double *q, const double *K, const double *V, int64_t L, int dh,
                double tau, double *out)
{
    for (int d = 0; d < dh; d++) out[d] = 0.0;
    if (L <= 0) return 0;
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    if (!s) return -2;
    double m = -INFINITY;
    for (int64_t t = 0; t < L; t++) {
        double acc = 0.0;
        for (int d = 0; d < dh; d++) acc += q[d] * K[t * dh + d];
        s[t] = tau * acc;
        if (s[t] > m) m = s[t];
    }
    double l = 0.0;
    for (int64_t t = 0; t < L; t++) {
        s[t] = exp(s[t] - m);
        l += s[t];
    }
    for (int64_t t = 0; t < L; t++) {
        double p = s[t] / l;
        for (int d = 0; d < dh; d++) out[d] += p * V[t * dh + d];
    }
    free(s);
    return 0;
}

/* Decode attention for a whole layer held in the cache layout
 *   codes  [B][Hkv][cap][dh*bits/8]   (bits 16: [B][Hkv][cap][dh] fp16)
 *   scales [B][Hkv][cap][dh/group]    fp16 (unused for bits 16)
 * q is [B][Hq][dh] (float values), lens[b] tokens are attended.
 * out is [B][Hq][dh] fp64.  tau <= 0 means 1/sqrt(dh). */
int kvqo_decode_layer(int B, int Hq, int Hkv, int dh, int cap,
                      const uint8_t *k_codes, const uint16_t *k_scales, int k_bits, int k_group,
                      const uint8_t *v_codes, const uint16_t *v_scales, int v_bits, int v_group,
                      const float *q, const int32_t *lens, double tau, double *out, int n_threads)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    if (tau <= 0.0) tau = 1.0 / sqrt((double)dh);
    /* one-byte codes: e4m3 and asymmetric INT8 */
    const int k1 = k_bits == KVQO_E4M3 || k_bits == KVQO_ASYM8;
    const int v1 = v_bits == KVQO_E4M3 || v_bits == KVQO_ASYM8;
    const int64_t krow = (k_bits == 16) ? (int64_t)dh * 2 : (k1 ? (int64_t)dh : (int64_t)dh * k_bits / 8);
    const int64_t vrow = (v_bits == 16) ? (int64_t)dh * 2 : (v1 ? (int64_t)dh : (int64_t)dh * v_bits / 8);
    /* fp16 values per row in the scale arrays: a pair per group when asymmetric */
    const int kng = (k_bits == 16) ? 0 : (dh / k_group) * (k_bits == KVQO_ASYM8 ? 2 : 1);
    const int vng = (v_bits == 16) ? 0 : (dh / v_group) * (v_bits == KVQO_ASYM8 ? 2 : 1);
    int rc = 0;
    (void)n_threads;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : rc)
#endif
    for (int bh = 0; bh < B * Hkv; bh++) {
        const int b = bh / Hkv, kvh = bh % Hkv;
        int64_t L = lens[b];
        if (L < 0) L = 0;
        if (L > cap) L = cap;
        double *Kd = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * dh);
        double *Vd = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * dh);
        double *qd = (double *)malloc(sizeof(double) * (size_t)dh);
        if (!Kd || !Vd || !qd) {
            rc |= 2;
        } else {
            const int64_t slab = (int64_t)bh * cap;
            rc |= kvqo_dequantize_rows(k_codes + slab * krow, k_scales ? k_scales + slab * kng : NULL,
                                       L, dh, k_group, k_bits, Kd) ? 1 : 0;
            rc |= kvqo_dequantize_rows(v_codes + slab * vrow, v_scales ? v_scales + slab * vng : NULL,
                                       L, dh, v_group, v_bits, Vd) ? 1 : 0;
            for (int g = 0; g < G; g++) {
                const int h = kvh * G + g;
                const float *qh = q + ((int64_t)b * Hq + h) * dh;
                for (int d = 0; d < dh; d++) qd[d] = (double)qh[d];
                rc |= kvqo_attend(qd, Kd, Vd, L, dh, tau, out + ((int64_t)b * Hq + h) * dh) ? 1 : 0;
            }
        }
        free(Kd);
        free(Vd);
        free(qd);
    }
    return rc ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* h-mode reconstruction                                                     */
/* ------------------------------------------------------------------------ */

/* h codes [n_tok][D*bits/8] with [n_tok][h_groups] fp16 scales (bits 16:
 * fp16 h).  W is bf16 [N][D].  For every token: h^ = dequant(h); if
 * round_bf16, h^ is rounded to bf16 (the GEMM operand); y = W h^ in fp64.
 * out_f64 [n_tok][N] (may be NULL) and out_f16 [n_tok][N] fp16 (may be NULL). */
int kvqo_h_reconstruct(const uint8_t *h_codes, const uint16_t *h_scales, int64_t n_tok, int D,
                       int h_groups, int h_bits, const uint16_t *w_bf16, int N, int round_bf16,
                       double *out_f64, uint16_t *out_f16, int n_threads)
{
    if (h_groups <= 0 || D % h_groups != 0) return -1;
    const int group = D / h_groups;
    double *W = (double *)malloc(sizeof(double) * (size_t)N * D);
    if (!W) return -2;
    for (int64_t i = 0; i < (int64_t)N * D; i++) W[i] = (double)kvqo_bf16_to_f32(w_bf16[i]);
    const int64_t row_bytes = (h_bits == 16) ? (int64_t)D * 2 : (int64_t)D * h_bits / 8;
    int rc = 0;
    (void)n_threads;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 16) reduction(| : rc)
#endif
    for (int64_t t = 0; t < n_tok; t++) {
        double *h = (double *)malloc(sizeof(double) * (size_t)D);
        if (!h) {
            rc |= 2;
            continue;
        }
        rc |= kvqo_dequantize_rows(h_codes + t * row_bytes, h_scales ? h_scales + t * h_groups : NULL,
                                   1, D, group, h_bits, h) ? 1 : 0;
        if (round_bf16)
            for (int i = 0; i < D; i++) h[i] = (double)kvqo_bf16_to_f32(kvqo_f32_to_bf16((float)h[i]));
        for (int n = 0; n < N; n++) {
            double acc = 0.0;
            const double *wr = W + (int64_t)n * D;
            for (int i = 0; i < D; i++) acc += wr[i] * h[i];
            if (out_f64) out_f64[t * N + n] = acc;
            if (out_f16) out_f16[t * N + n] = kvqo_f64_to_f16(acc);
        }
        free(h);
    }
    free(W);
    return rc ? -1 : 0;
}

/* h-mode decode by query absorption (an algebraic rewrite of the
 * reconstruction path of the TinyLoop page, "運作原理": K = W_k h and
 * V = W_v h are linear in h, so q . K_t = (W_k,j^T q) . h_t and
 * sum_t p_t V_t = W_v,j (sum_t p_t h_t) for KV head j).  For every sequence b
 * and query head h (KV head j = h / G), all in fp64 with h^ dequantised
 * exactly and W the bf16 values:
 *   qa   = sum_i q[i] W[j Dh + i][:]              (W_k rows of head j)
 *   s_t  = tau qa . h^_t,  p = softmax(s) over t < lens[b]
 *   ob   = sum_t p_t h^_t
 *   out[i] = sum_d W[Hkv Dh + j Dh + i][d] ob[d]  (W_v rows of head j)
 * No rounding of h^ to bf16 nor of K/V to fp16: the result is the
 * reconstruction attention in exact arithmetic.  h codes [B][cap][row],
 * scales [B][cap][h_groups]; q float [B][Hq][Dh]; W bf16 [2 Hkv Dh][D];
 * out fp64 [B][Hq][Dh]; tau <= 0 means 1/sqrt(Dh); an empty sequence gives
 * zeros. */
int kvqo_h_absorbed_decode(int B, int Hq, int Hkv, int Dh, int D, int cap, const uint8_t *h_codes,
                           const uint16_t *h_scales, int h_bits, int h_groups,
                           const uint16_t *w_bf16, const float *q, const int32_t *lens, double tau,
                           double *out, int n_threads)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || Hkv * Dh != D || h_groups <= 0 || D % h_groups != 0)
        return -1;
    const int G = Hq / Hkv;
    const int group = D / h_groups;
    if (tau <= 0.0) tau = 1.0 / sqrt((double)Dh);
    const int64_t row_bytes = (h_bits == 16) ? (int64_t)D * 2 : (int64_t)D * h_bits / 8;
    int rc = 0;
    (void)n_threads;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : rc)
#endif
    for (int bh = 0; bh < B * Hq; bh++) {
        const int b = bh / Hq, h = bh % Hq, j = h / G;
        int64_t L = lens[b];
        if (L < 0) L = 0;
        if (L > cap) L = cap;
        double *o = out + (int64_t)bh * Dh;
        for (int i = 0; i < Dh; i++) o[i] = 0.0;
        if (L == 0) continue;
        double *H = (double *)malloc(sizeof(double) * (size_t)L * D);
        double *qa = (double *)malloc(sizeof(double) * (size_t)D);
        double *ob = (double *)malloc(sizeof(double) * (size_t)D);
        double *sc = (double *)malloc(sizeof(double) * (size_t)L);
        if (!H || !qa || !ob || !sc) {
            rc |= 2;
        } else {
            const int64_t slab = (int64_t)b * cap;
            rc |= kvqo_dequantize_rows(h_codes + slab * row_bytes,
                                       h_scales ? h_scales + slab * h_groups : NULL, L, D, group,
                                       h_bits, H) ? 1 : 0;
            const float *qh = q + (int64_t)bh * Dh;
            for (int d = 0; d < D; d++) {
                double acc = 0.0;
                for (int i = 0; i < Dh; i++)
                    acc += (double)qh[i] * (double)kvqo_bf16_to_f32(w_bf16[(int64_t)(j * Dh + i) * D + d]);
                qa[d] = acc;
            }
            double m = -INFINITY;
            for (int64_t t = 0; t < L; t++) {
                double acc = 0.0;
                for (int d = 0; d < D; d++) acc += qa[d] * H[t * D + d];
                sc[t] = tau * acc;
                if (sc[t] > m) m = sc[t];
            }
            double l = 0.0;
            for (int64_t t = 0; t < L; t++) {
                sc[t] = exp(sc[t] - m);
                l += sc[t];
            }
            for (int d = 0; d < D; d++) ob[d] = 0.0;
            for (int64_t t = 0; t < L; t++) {
                const double p = sc[t] / l;
                for (int d = 0; d < D; d++) ob[d] += p * H[t * D + d];
            }
            for (int i = 0; i < Dh; i++) {
                const uint16_t *wr = w_bf16 + (int64_t)(Hkv * Dh + j * Dh + i) * D;
                double acc = 0.0;
                for (int d = 0; d < D; d++) acc += (double)kvqo_bf16_to_f32(wr[d]) * ob[d];
                o[i] = acc;
            }
        }
        free(H);
        free(qa);
        free(ob);
        free(sc);
    }
    return rc ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Bytes per token per layer                                                 */
/* ------------------------------------------------------------------------ */

/* TinyLoop docs, "記憶體公式": FP16 KV 2*D*2; INT8 KV 2*D*1 + 2*n_heads*2;
 * FP16 h D*2; INT8 h D + n_heads*2; INT4 h D/2 + n_heads*2.  Generalised to
 * separate K/V widths and scale groups (KVSplit): each stored tensor costs
 * Hkv*dh*bits/8 code bytes plus Hkv*(dh/group) fp16 scales (none at 16 bits).
 * mode 0 = K/V cache, mode 1 = h cache. */
int kvqo_bytes_per_token_layer(int mode, int n_kv_heads, int head_dim, int k_bits, int v_bits,
                               int k_group, int v_group, int d_model, int h_bits, int h_groups,
                               uint64_t *out)
{
    uint64_t b = 0;
    if (mode == 0) {
        const int bits[2] = {k_bits, v_bits};
        const int grp[2] = {k_group, v_group};
        for (int i = 0; i < 2; i++) {
            uint64_t elems = (uint64_t)n_kv_heads * head_dim;
            b += elems * bits[i] / 8;
            if (bits[i] != 16) b += (uint64_t)n_kv_heads * (head_dim / grp[i]) * 2;
        }
    } else if (mode == 1) {
        b = (uint64_t)d_model * h_bits / 8;
        if (h_bits != 16) b += (uint64_t)h_groups * 2;
    } else {
        return -1;
    }
    *out = b;
    return 0;
}
