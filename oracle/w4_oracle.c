/*
 * w4_oracle.c -- plain, slow CPU oracle for group-wise INT4 weight quantization
 * and the W4A16 product.  TEST INFRASTRUCTURE ONLY: it exists so that the CUDA
 * library can be checked against an obviously-correct restatement of the
 * method.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg load it; the product path never does.  It shares no code,
 * header or table with the CUDA library.
 *
 * Sources (web pages on LLM quantization; "page N" below):
 *   page 5  ai-infra.cypggs.com .../model-quantization/02-core-ideas, section 2.2
 *           "rounding": symmetric q = clip(round(x/s), -2^(b-1), 2^(b-1)-1) with
 *           s = max|x|/(2^(b-1)-1); asymmetric q = clip(round(x/s)+zp, 0, 2^b-1)
 *           with s = (max-min)/(2^b-1), zp = round(-min/s); dequantize
 *           x^ = (q-zp)*s; default rounding is round-to-nearest-even.
 *   page 2  learn.longtimenohack.com .../quantization.html, "group quantization":
 *           groups of g = 128 weights along a row share one fp16 scale and an
 *           integer zero-point.
 *   page 3  blog.freezetheflame.cc .../quantization-deep-dive.html, section 2.2
 *           (per-group scales have shape [C_out, num_groups]) and section 5.3
 *           (the smoothing vector s is folded into the weights offline, W*s).
 *   page 5  section 2.4: X' = X/s, W' = W*diag(s), X'W'^T == XW^T.
 *   page 5  section 2.1: the E2M1 value set.
 *
 * Readings where the pages leave a step open (each is also listed in the
 * design notes of the repository):
 *   b = 4.  Symmetric: s32 = fl32(amax/7), codes q in [-8,7] stored as u = q+8.
 *   Asymmetric: min and max are taken with 0 included, s32 = fl32((mx-mn)/15),
 *   zp = clip(rint(fl32(-mn/s16)), 0, 15), u = clip(rint(fl32(w/s16))+zp, 0, 15).
 *   The stored scale is s16 = fp16_rne(s32) (saturated to 65504) and both zp
 *   and the codes are derived from float(s16).  If s16 == 0 every code is the
 *   zero code (u = 8 symmetric; zp = 0, u = 0 asymmetric).
 *   Dequantized weight w^ = bf16_rne(float(u-zp) * float(s16)) (symmetric zp=8).
 *   Product Y[m][n] = sum_k x[m][k] * w^[n][k] in fp64.
 *
 * Arithmetic: IEEE binary32 with round-to-nearest-even, one rounding per
 * operation (compiled with -ffp-contract=off, no fast-math); the conversions to
 * fp16 and bf16 are written out below from the formats' definitions.
 *
 * Packed layout (the library's documented layout, restated here):
 *   qweight[n][c], c = k/8: bits [4i,4i+4) hold element 8c+2i and bits
 *   [16+4i,16+4i+4) hold element 8c+2i+1, for i = 0..3.
 *   scales[n][j]: fp16 bits of group j = k/g.
 *   qzeros[n][c], c = j/8: bits [4(j%8), 4(j%8)+4) hold zp of group j; unused
 *   nibbles are 0.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <fenv.h>

#if defined(__FAST_MATH__)
#error "the oracle must be compiled without fast-math"
#endif

/* ------------------------------------------------------------------------ */
/* Floating-point format conversions, from the IEEE 754 binary16 definition  */
/* (1 sign, 5 exponent bits with bias 15, 10 fraction bits, subnormals with  */
/* quantum 2^-24) and the bfloat16 definition (the upper half of binary32:    */
/* 1 sign, 8 exponent bits with bias 127, 7 fraction bits).                   */
/* ------------------------------------------------------------------------ */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* Round the finite nonzero magnitude m*2^E to p significant bits with the
 * quantum bounded below by 2^qmin, ties to even.  Returns r and sets *qe so
 * that the rounded magnitude is r*2^(*qe) with r < 2^p, or r == 2^p exactly
 * after a carry (the caller renormalises). */
static uint64_t round_sig(uint64_t m, int E, int p, int qmin, int *qe)
{
    int L = E + (63 - __builtin_clzll(m));      /* floor(log2(m*2^E)) */
    int q = L - (p - 1);
    if (q < qmin) q = qmin;
    int sh = q - E;                             /* low bits to drop   */
    uint64_t r;
    if (sh <= 0) {
        r = m << (-sh);
    } else if (sh >= 64) {
        r = 0;
    } else {
        uint64_t keep = m >> sh;
        uint64_t rem = m & ((1ull << sh) - 1);
        uint64_t half = 1ull << (sh - 1);
        r = keep + ((rem > half) || (rem == half && (keep & 1)));
    }
    *qe = q;
    return r;
}

/* float -> IEEE binary16 bits, round to nearest even; overflow gives inf. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t x = f32_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ex = (x >> 23) & 0xFFu, fr = x & 0x7FFFFFu;
    if (ex == 0xFFu) return (uint16_t)(sign | 0x7C00u | (fr ? 0x0200u : 0u));
    if (ex == 0 && fr == 0) return sign;
    uint64_t m = ex ? (fr | 0x800000u) : fr;
    int E = ex ? (int)ex - 150 : -149;
    int qe;
    uint64_t r = round_sig(m, E, 11, -24, &qe);
    if (r == 0) return sign;
    if (r < 1024u) return (uint16_t)(sign | r);            /* subnormal, qe = -24 */
    if (r == 2048u) { r = 1024u; qe += 1; }                 /* carry into exponent */
    int bexp = qe + 25;                                     /* (r/2^10)*2^(qe+10)  */
    if (bexp >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | ((uint32_t)bexp << 10) | (uint32_t)(r - 1024u));
}

float orc_f16_to_f32(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)f, -24);
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(1024 + f), e - 25);
    return (float)(s ? -v : v);
}

/* float -> bfloat16 bits, round to nearest even; overflow gives inf. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t x = f32_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ex = (x >> 23) & 0xFFu, fr = x & 0x7FFFFFu;
    if (ex == 0xFFu) return (uint16_t)(sign | 0x7F80u | (fr ? 0x0040u : 0u));
    if (ex == 0 && fr == 0) return sign;
    uint64_t m = ex ? (fr | 0x800000u) : fr;
    int E = ex ? (int)ex - 150 : -149;
    int qe;
    uint64_t r = round_sig(m, E, 8, -133, &qe);
    if (r == 0) return sign;
    if (r < 128u) return (uint16_t)(sign | r);              /* subnormal, qe = -133 */
    if (r == 256u) { r = 128u; qe += 1; }
    int bexp = qe + 134;                                    /* (r/2^7)*2^(qe+7)    */
    if (bexp >= 255) return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | ((uint32_t)bexp << 7) | (uint32_t)(r - 128u));
}

float orc_bf16_to_f32(uint16_t b)
{
    uint32_t x = (uint32_t)b << 16;
    float f;
    memcpy(&f, &x, 4);
    return f;
}

/* Stored scale: fp16 of s32, saturated at the largest finite fp16 (65504). */
static uint16_t scale_to_f16(float s32)
{
    if (s32 > 65504.0f) return 0x7BFFu;
    return orc_f32_to_f16(s32);
}

static float clipf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ------------------------------------------------------------------------ */
/* One group (page 5 section 2.2 formulas, b = 4).                           */
/*   w      : g folded weights w' (fp32)                                      */
/*   mode   : 0 symmetric, 1 asymmetric                                       */
/* outputs  : s16 (fp16 bits), zp (8 in symmetric mode), u[g] codes 0..15      */
/* ------------------------------------------------------------------------ */
void orc_quant_group(const float *w, int64_t g, int mode, uint16_t *s16_out, int *zp_out, uint8_t *u)
{
    if (mode == 0) {
        float amax = 0.0f;                                   /* max |w'| */
        for (int64_t i = 0; i < g; ++i) {
            float a = fabsf(w[i]);
            if (a > amax) amax = a;
        }
        float s32 = amax / 7.0f;                             /* s = max|x| / (2^(b-1)-1) */
        uint16_t s16 = scale_to_f16(s32);
        float d = orc_f16_to_f32(s16);
        for (int64_t i = 0; i < g; ++i) {
            float q = 0.0f;
            if (d != 0.0f) q = clipf(nearbyintf(w[i] / d), -8.0f, 7.0f);   /* clip(round(x/s)) */
            u[i] = (uint8_t)((int)q + 8);                    /* offset-binary storage */
        }
        *s16_out = s16;
        *zp_out = 8;
    } else {
        float mn = 0.0f, mx = 0.0f;                          /* range extended to include 0 */
        for (int64_t i = 0; i < g; ++i) {
            if (w[i] < mn) mn = w[i];
            if (w[i] > mx) mx = w[i];
        }
        float range = mx - mn;
        float s32 = range / 15.0f;                           /* s = (max-min)/(2^b-1) */
        uint16_t s16 = scale_to_f16(s32);
        float d = orc_f16_to_f32(s16);
        int zp = 0;
        if (d != 0.0f) zp = (int)clipf(nearbyintf(-mn / d), 0.0f, 15.0f);   /* zp = round(-min/s) */
        for (int64_t i = 0; i < g; ++i) {
            float q = 0.0f;
            if (d != 0.0f) q = clipf(nearbyintf(w[i] / d) + (float)zp, 0.0f, 15.0f);
            u[i] = (uint8_t)q;
        }
        *s16_out = s16;
        *zp_out = zp;
    }
}

/* ------------------------------------------------------------------------ */
/* Whole matrix: fold (optional), group quantize, pack.  Rows [r0, r1).       */
/* W bf16 bits [N,K] row-major; s fp32 [K] or NULL.                           */
/* Returns 0 on success, nonzero on bad arguments.                            */
/* ------------------------------------------------------------------------ */
int orc_quant_pack_rows(const uint16_t *W, int64_t N, int64_t K, int64_t g, int mode, const float *s,
                        int64_t r0, int64_t r1, uint32_t *qweight, uint16_t *scales, uint32_t *qzeros)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || K % 8 != 0 || r0 < 0 || r1 > N || r0 > r1) return 1;
    if (fegetround() != FE_TONEAREST) return 2;
    int64_t G = K / g, ZW = (G + 7) / 8;
    float wf[512];
    uint8_t u[512];
    if (g > 512) return 3;
    for (int64_t n = r0; n < r1; ++n) {
        const uint16_t *row = W + n * K;
        uint32_t *qrow = qweight + n * (K / 8);
        memset(qrow, 0, (size_t)(K / 8) * 4);
        if (mode == 1) memset(qzeros + n * ZW, 0, (size_t)ZW * 4);
        for (int64_t j = 0; j < G; ++j) {
            for (int64_t i = 0; i < g; ++i) {
                int64_t k = j * g + i;
                float w = orc_bf16_to_f32(row[k]);
                wf[i] = s ? w * s[k] : w;                    /* w' = w * s[k] (fold) */
            }
            uint16_t s16;
            int zp;
            orc_quant_group(wf, g, mode, &s16, &zp, u);
            scales[n * G + j] = s16;
            if (mode == 1) qzeros[n * ZW + j / 8] |= (uint32_t)zp << (4 * (j % 8));
            for (int64_t i = 0; i < g; ++i) {
                int64_t k = j * g + i;
                int64_t c = k / 8, e = k % 8;
                int sh = (e % 2 == 0) ? 4 * (int)(e / 2) : 16 + 4 * (int)(e / 2);
                qrow[c] |= (uint32_t)u[i] << sh;
            }
        }
    }
    return 0;
}

/* Code u of element (n,k) and zero-point of its group, read back from the
 * packed layout. */
static int code_at(const uint32_t *qweight, int64_t K, int64_t n, int64_t k)
{
    uint32_t word = qweight[n * (K / 8) + k / 8];
    int64_t e = k % 8;
    int sh = (e % 2 == 0) ? 4 * (int)(e / 2) : 16 + 4 * (int)(e / 2);
    return (int)((word >> sh) & 0xFu);
}

static int zp_at(const uint32_t *qzeros, int64_t G, int mode, int64_t n, int64_t j)
{
    if (mode == 0) return 8;
    int64_t ZW = (G + 7) / 8;
    return (int)((qzeros[n * ZW + j / 8] >> (4 * (j % 8))) & 0xFu);
}

/* Dequantize rows [r0,r1): w^ = bf16_rne(float(u - zp) * float(s16)) (page 5 x^ = (q-zp)*s). */
int orc_dequant_rows(const uint32_t *qweight, const uint16_t *scales, const uint32_t *qzeros,
                     int64_t N, int64_t K, int64_t g, int mode, int64_t r0, int64_t r1, uint16_t *what)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || K % 8 != 0 || r0 < 0 || r1 > N || r0 > r1) return 1;
    int64_t G = K / g;
    for (int64_t n = r0; n < r1; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t j = k / g;
            float d = orc_f16_to_f32(scales[n * G + j]);
            int D = code_at(qweight, K, n, k) - zp_at(qzeros, G, mode, n, j);
            what[(n - r0) * K + k] = orc_f32_to_bf16((float)D * d);
        }
    }
    return 0;
}

/* Same, without the final bf16 rounding: the exact fp32 product (u-zp)*s16. */
int orc_dequant_rows_f32(const uint32_t *qweight, const uint16_t *scales, const uint32_t *qzeros,
                         int64_t N, int64_t K, int64_t g, int mode, int64_t r0, int64_t r1, float *what)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || K % 8 != 0 || r0 < 0 || r1 > N || r0 > r1) return 1;
    int64_t G = K / g;
    for (int64_t n = r0; n < r1; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t j = k / g;
            float d = orc_f16_to_f32(scales[n * G + j]);
            int D = code_at(qweight, K, n, k) - zp_at(qzeros, G, mode, n, j);
            what[(n - r0) * K + k] = (float)D * d;
        }
    }
    return 0;
}

/* Y[m][c] = sum_k double(x[m][k]) * double(w^[c][k]): X bf16 [M,K], W^ bf16
 * [C,K] (the dequantized rows of the output channels wanted), Y fp64 [M,C]. */
void orc_gemm_f64(const uint16_t *X, int64_t M, int64_t K, const uint16_t *What, int64_t C, double *Y)
{
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t *xr = X + m * K;
        for (int64_t c = 0; c < C; ++c) {
            const uint16_t *wr = What + c * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)orc_bf16_to_f32(xr[k]) * (double)orc_bf16_to_f32(wr[k]);
            Y[m * C + c] = acc;
        }
    }
}

/* E2M1 (FP4): 1 sign bit, 2 exponent bits with bias 1, 1 fraction bit;
 * exponent field 0 encodes the subnormals 0 and 0.5 (page 5 section 2.1). */
float orc_e2m1_decode(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, f = code & 1;
    double v = (e == 0) ? ldexp((double)f, -1) : ldexp(1.0 + 0.5 * f, e - 1);
    return (float)(s ? -v : v);
}

/* ------------------------------------------------------------------------ */
/* FP4 block-scaled weights (NVFP4 and MXFP4).                               */
/*                                                                           */
/* Page 2 (learn.longtimenohack.com .../quantization.html, the Blackwell FP4  */
/* paragraph and its teaching snippet): E2M1 values, blocks of 16 weights     */
/* sharing one FP8 E4M3 scale, amax mapped to the E2M1 maximum 6, 4 + 8/16 =  */
/* 4.5 bits per weight.  Page 3 (blog.freezetheflame.cc .../quantization-     */
/* deep-dive.html, section 4.3): MXFP4, blocks of 32 sharing an E8M0 scale,   */
/* two FP4 values per byte.  Page 5 (ai-infra.cypggs.com .../02-core-ideas,   */
/* section 2.1): the E2M1 value set and the E4M3 format (1+4+3, max 448,      */
/* S.1111.111 is NaN).                                                        */
/*                                                                           */
/* Readings where the pages leave a step open:                               */
/*   NVFP4: s = e4m3_rn(fl32(amax / 6)), codes e2m1_rn(fl32(w / s)); the      */
/*     snippet's second factor 6.0 is garbled (it would map amax to 36) and   */
/*     is left out; a block whose s is 0 gets all-zero codes.                 */
/*   MXFP4: the pages give no exponent rule; the shared scale is            */
/*     2^(floor(log2 amax) - 2), the OCP Microscaling rule with the E2M1     */
/*     maximum exponent 2, clamped to the E8M0 range [-127, 127]; an all-    */
/*     zero block gets 2^-127 and zero codes.                                 */
/*   Both: elements round to nearest E2M1 value, ties to the even fraction    */
/*     bit, magnitudes above 6 saturate to 6; scales saturate too (E4M3 at    */
/*     448).  Codes pack two per byte, element 2i in the low nibble.          */
/*   Dequantized weight w^ = e2m1(code) * scale, exact in fp32 (at most 6     */
/*   significant bits), so also exact in bf16 within bf16's range.           */
/* ------------------------------------------------------------------------ */

/* E4M3 (OCP FP8 "FN"): 1 sign bit, 4 exponent bits with bias 7, 3 fraction
 * bits; exponent field 0 encodes subnormals f * 2^-9; no infinity; the
 * all-ones magnitude S.1111.111 is NaN, so the largest finite value is 448. */
float orc_e4m3_decode(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, f = code & 7;
    double v;
    if (e == 15 && f == 7) v = NAN;
    else if (e == 0) v = ldexp((double)f, -9);
    else v = ldexp((double)(8 + f), e - 10);
    return (float)(s ? -v : v);
}

/* float -> E4M3 code, round to nearest even; finite magnitudes that round
 * above 448 (and infinities) saturate to 448, NaN stays NaN. */
int orc_f32_to_e4m3_sat(float f)
{
    uint32_t x = f32_bits(f);
    int sign = (x >> 31) ? 0x80 : 0;
    uint32_t ex = (x >> 23) & 0xFFu, fr = x & 0x7FFFFFu;
    if (ex == 0xFFu) return fr ? (sign | 0x7F) : (sign | 0x7E);
    if (ex == 0 && fr == 0) return sign;
    uint64_t m = ex ? (fr | 0x800000u) : fr;
    int E = ex ? (int)ex - 150 : -149;
    int qe;
    uint64_t r = round_sig(m, E, 4, -9, &qe);
    if (r == 0) return sign;
    if (r < 8u) return sign | (int)r;                       /* subnormal, qe = -9     */
    if (r == 16u) { r = 8u; qe += 1; }                      /* carry into exponent    */
    int bexp = qe + 10;                                     /* r * 2^qe, r in [8, 16) */
    if (bexp > 15 || (bexp == 15 && r - 8u == 7u)) return sign | 0x7E;
    return sign | (bexp << 3) | (int)(r - 8u);
}

/* float -> E2M1 code, round to nearest even (ties to the even fraction bit);
 * magnitudes above 6 saturate to 6.  Exponent field 0 holds 0 and 0.5. */
int orc_f32_to_e2m1_sat(float f)
{
    uint32_t x = f32_bits(f);
    int sign = (x >> 31) ? 8 : 0;
    uint32_t ex = (x >> 23) & 0xFFu, fr = x & 0x7FFFFFu;
    if (ex == 0xFFu) return sign | 7;
    if (ex == 0 && fr == 0) return sign;
    uint64_t m = ex ? (fr | 0x800000u) : fr;
    int E = ex ? (int)ex - 150 : -149;
    int qe;
    uint64_t r = round_sig(m, E, 2, -1, &qe);
    if (r == 0) return sign;
    if (r < 2u) return sign | (int)r;                       /* 0.5, qe = -1           */
    if (r == 4u) { r = 2u; qe += 1; }
    int e = qe + 2;                                         /* r * 2^qe, r in {2, 3}  */
    if (e > 3) return sign | 7;
    return sign | (e << 1) | (int)(r - 2u);
}

/* E8M0: the power of two 2^(code - 127), code in [0, 254] (255 is NaN). */
float orc_e8m0_decode(int code)
{
    if ((code & 0xFF) == 0xFF) return NAN;
    return (float)ldexp(1.0, (code & 0xFF) - 127);
}

/* Block-scaled FP4 quantization of W (bf16 [N, K], K a multiple of the block).
 * kind 0 = NVFP4 (block 16, E4M3 scales), 1 = MXFP4 (block 32, E8M0 scales).
 * codes: uint8 [N, K/2], scales: uint8 [N, K/block]. */
int orc_fp4_quant_rows(const uint16_t *W, int64_t N, int64_t K, int kind, uint8_t *codes, uint8_t *scales)
{
    const int64_t B = kind == 0 ? 16 : 32;
    if (K % B != 0 || (kind != 0 && kind != 1)) return -1;
    memset(codes, 0, (size_t)(N * (K / 2)));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < K / B; ++b) {
            const uint16_t *w = W + n * K + b * B;
            float amax = 0.0f;
            for (int64_t i = 0; i < B; ++i) {
                float a = fabsf(orc_bf16_to_f32(w[i]));
                if (a > amax) amax = a;
            }
            float sc;
            int scode;
            if (kind == 0) {
                volatile float t = amax / 6.0f;                 /* one IEEE division */
                scode = orc_f32_to_e4m3_sat(t);
                sc = orc_e4m3_decode(scode);
            } else {
                int e = -127;
                if (amax > 0.0f) {
                    int ex;
                    frexp((double)amax, &ex);               /* amax = f 2^ex, f in [0.5, 1) */
                    e = (ex - 1) - 2;                       /* floor(log2 amax) - 2          */
                    if (e < -127) e = -127;
                    if (e > 127) e = 127;
                }
                scode = e + 127;
                sc = orc_e8m0_decode(scode);
            }
            scales[n * (K / B) + b] = (uint8_t)scode;
            for (int64_t i = 0; i < B; ++i) {
                int q = 0;
                if (sc > 0.0f) {
                    volatile float t = orc_bf16_to_f32(w[i]) / sc;   /* one IEEE division */
                    q = orc_f32_to_e2m1_sat(t);
                }
                const int64_t k = b * B + i;
                codes[n * (K / 2) + k / 2] |= (uint8_t)(q << (4 * (k & 1)));
            }
        }
    }
    return 0;
}

/* w^[n][k] = e2m1(code) * scale, fp32 [N, K]. */
int orc_fp4_dequant_rows(const uint8_t *codes, const uint8_t *scales, int64_t N, int64_t K, int kind, float *out)
{
    const int64_t B = kind == 0 ? 16 : 32;
    if (K % B != 0 || (kind != 0 && kind != 1)) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            const int q = (codes[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 15;
            const int sc = scales[n * (K / B) + k / B];
            const double s = kind == 0 ? (double)orc_e4m3_decode(sc) : (double)orc_e8m0_decode(sc);
            out[n * K + k] = (float)((double)orc_e2m1_decode(q) * s);
        }
    return 0;
}

/* MXFP8 activations for the block-scaled tensor-core product (page 3 section
 * 4.3: FP4 for the weights, activations kept at FP8; MX blocks of 32 share an
 * E8M0 scale).  Reading: the OCP Microscaling rule with the E4M3 maximum
 * exponent 8 (448 = 1.75 * 2^8): scale 2^(floor(log2 amax) - 8) clamped to
 * [-127, 127], elements e4m3_rn(fl32(x / scale)) saturating at 448; an
 * all-zero block gets 2^-127 and zero codes.  X: bf16 [M, K]; codes: uint8
 * [M, K] (E4M3); scales: uint8 [M, K/32] (E8M0). */
int orc_mxfp8_quant_rows(const uint16_t *X, int64_t M, int64_t K, uint8_t *codes, uint8_t *scales)
{
    if (K % 32 != 0) return -1;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < K / 32; ++b) {
            const uint16_t *x = X + m * K + b * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(orc_bf16_to_f32(x[i]));
                if (a > amax) amax = a;
            }
            int e = -127;
            if (amax > 0.0f) {
                int ex;
                frexp((double)amax, &ex);
                e = (ex - 1) - 8;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            scales[m * (K / 32) + b] = (uint8_t)(e + 127);
            const float sc = orc_e8m0_decode(e + 127);
            for (int i = 0; i < 32; ++i) {
                volatile float t = orc_bf16_to_f32(x[i]) / sc;      /* one IEEE division */
                codes[m * K + b * 32 + i] = (uint8_t)orc_f32_to_e4m3_sat(t);
            }
        }
    }
    return 0;
}

/* x^[m][k] = e4m3(code) * scale, fp32 [M, K] (exact). */
int orc_mxfp8_dequant_rows(const uint8_t *codes, const uint8_t *scales, int64_t M, int64_t K, float *out)
{
    if (K % 32 != 0) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k)
            out[m * K + k] = (float)((double)orc_e4m3_decode(codes[m * K + k]) *
                                     (double)orc_e8m0_decode(scales[m * (K / 32) + k / 32]));
    return 0;
}
