/*
 * qf_oracle.c -- the ORACLE for deployment-aligned simulated quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, scalar CPU statement
 * of what the hot path computes.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load it.  The product path (the CUDA library)
 * shares no code, header, table or constant generator with it and never calls it.
 *
 * Source of the method: "QATFactory: A Versatile, Deployment-Aligned Framework
 * for Quantization-aware Training and Distillation of LLMs", project page
 * (weilixu.com/QATFactory-web):
 *   [M-QDQ]   Method, "Framework overview": training quantizes and at once
 *             dequantizes in the forward pass, so the model computes with the
 *             numbers inference will use; gradients pass straight through to the
 *             full-precision weights (a straight-through estimator).
 *   [M-NUM]   Method, "Numerics": the serving engine defines the values, block
 *             sizes and scaling rules; for NVFP4, projections the engine runs as
 *             one fused GEMM (QKV, gate/up) use a common tensor scale, while
 *             MXFP4 and Q4_K have no tensor-level scale at all.
 *   [T-FMT]   "Supported formats" table: NVFP4 = E2M1 elements, block 16, E4M3
 *             block scale + FP32 tensor scale, symmetric, 4.50 bits/weight;
 *             MXFP4 = E2M1, block 32, E8M0 block scale, symmetric, 4.25 b/w;
 *             Q4_K = unsigned INT4, block 32 in a 256 super-block, 6-bit block
 *             scales + FP16 super-block scales, asymmetric, 4.50 b/w.  The
 *             bits-per-weight figures count the codes plus the scale bytes.
 *   [M-EXP]   Method, "QARL" and "Export": weights are written in the byte layout
 *             the engine loads; the NVFP4 activation amax is kept from training.
 *   [M-QAD]   Method, "QAD": MoE experts are quantized in separate passes.
 *
 * Arithmetic: the pages fix FP32 as the tensor-scale type [T-FMT]; every scale
 * and element step below is IEEE binary32 with round-to-nearest-even and no
 * fused multiply-add (build with -ffp-contract=off, no fast-math).  Each step is
 * one named IEEE operation so the order of rounding is the one written here.
 * Conversions between number formats are written from the formats' bit-level
 * definitions (exact arithmetic in binary64, then one rounding).
 *
 * Readings where the pages are silent (rounding mode, scale derivation,
 * saturation, Q4_K fitting, byte layouts) are stated at each function.
 * Bytes: BF16 and FP16 values travel as uint16_t bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#if defined(__FAST_MATH__)
#error "the oracle must be built without fast-math"
#endif

/* ------------------------------------------------------------------------ */
/* bit views                                                                 */
/* ------------------------------------------------------------------------ */
static float f32_of_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_of_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* ------------------------------------------------------------------------ */
/* Generic "round a magnitude onto a binary floating-point grid".            */
/*                                                                           */
/* A format with `mbits` stored mantissa bits and minimum normal exponent    */
/* `emin` represents, around a magnitude a, the multiples of                 */
/* quantum = 2^(max(floor(log2 a), emin) - mbits).  Rounding to nearest with */
/* ties to even means: n = a / quantum (exact in binary64, because a is a    */
/* binary32 value and quantum a power of two), then the integer nearest to n */
/* with ties to the even integer.  An even integer multiple is exactly an    */
/* even stored mantissa, so this is IEEE round-to-nearest-even.              */
/* Returns the rounded magnitude as a double (exact).                        */
/* ------------------------------------------------------------------------ */
static double round_to_grid(double a, int mbits, int emin)
{
    if (a == 0.0) return 0.0;
    int k;
    (void)frexp(a, &k);            /* a = m * 2^k, m in [0.5, 1) -> floor(log2 a) = k-1 */
    int e = k - 1;
    if (e < emin) e = emin;        /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, e - mbits);
    double n = a / quantum;        /* exact */
    double fl = floor(n);
    double frac = n - fl;          /* exact */
    double r;
    if (frac > 0.5) r = fl + 1.0;
    else if (frac < 0.5) r = fl;
    else r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;   /* tie: to the even multiple */
    return r * quantum;            /* exact (may carry into the next binade) */
}

/* ------------------------------------------------------------------------ */
/* BF16: the upper half of a binary32 (8 exponent bits, 7 mantissa bits).    */
/* ------------------------------------------------------------------------ */
float qfo_bf16_to_f32(uint16_t h) { return f32_of_bits((uint32_t)h << 16); }

/* binary32 -> BF16, round to nearest even, finite inputs (overflow -> inf). */
uint16_t qfo_f32_to_bf16(float f)
{
    uint32_t sign = bits_of_f32(f) & 0x80000000u;
    double a = fabs((double)f);
    double r = round_to_grid(a, 7, -126);
    if (r >= 0x1p128) return (uint16_t)((sign >> 16) | 0x7F80u);    /* +-inf */
    float rf = (float)r;                                             /* exact */
    return (uint16_t)((bits_of_f32(rf) | sign) >> 16);
}

/* ------------------------------------------------------------------------ */
/* FP16 (IEEE binary16): 5 exponent bits (bias 15), 10 mantissa bits.        */
/* ------------------------------------------------------------------------ */
float qfo_f16_to_f32(uint16_t h)
{
    int s = (h >> 15) & 1, E = (h >> 10) & 31, M = h & 1023;
    double v;
    if (E == 0) v = ldexp((double)M, -24);
    else if (E == 31) v = M ? NAN : INFINITY;
    else v = ldexp(1024.0 + M, E - 25);
    return (float)(s ? -v : v);
}

/* binary32 -> FP16, round to nearest even including subnormals. */
uint16_t qfo_f32_to_f16(float f)
{
    uint16_t sign = (bits_of_f32(f) >> 16) & 0x8000u;
    double a = fabs((double)f);
    double r = round_to_grid(a, 10, -14);
    if (r >= 65536.0) return sign | 0x7C00u;                         /* overflow -> inf */
    if (r == 0.0) return sign;
    int k;
    (void)frexp(r, &k);
    int e = k - 1;
    if (e < -14) return sign | (uint16_t)(r * 0x1p24);               /* subnormal */
    uint16_t E = (uint16_t)(e + 15);
    uint16_t M = (uint16_t)(ldexp(r, -e) * 1024.0 - 1024.0);
    return sign | (uint16_t)(E << 10) | M;
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit, no inf/NaN.      */
/* Magnitudes by 3-bit code: 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Code bit 3 = sign. */
/* [T-FMT] "Element: E2M1 (FP4)" for NVFP4 and MXFP4.                        */
/* ------------------------------------------------------------------------ */
float qfo_e2m1_to_f32(uint8_t c)
{
    int s = (c >> 3) & 1, E = (c >> 1) & 3, M = c & 1;
    double v = (E == 0) ? 0.5 * M : ldexp(1.0 + 0.5 * M, E - 1);
    return (float)(s ? -v : v);
}

/* binary32 -> E2M1, round to nearest even, saturating to +-6 ("satfinite").
 * Reading: the sign bit of the code is the sign bit of the input, so negative
 * values that round to zero give the code 0x8 (negative zero).  The input
 * must not be NaN (the callers never produce one). */
uint8_t qfo_e2m1_from_f32(float q)
{
    uint8_t sign = (bits_of_f32(q) >> 31) ? 8 : 0;
    double a = fabs((double)q);
    double r = round_to_grid(a, 1, 0);
    if (r > 6.0) r = 6.0;                                            /* satfinite */
    uint8_t mag;
    if (r < 1.0) mag = (uint8_t)(r * 2.0);                           /* 0 or 0.5 */
    else {
        int k; (void)frexp(r, &k);
        int e = k - 1;                                               /* 0..2 */
        mag = (uint8_t)(((e + 1) << 1) | (ldexp(r, -e) > 1.0 ? 1 : 0));
    }
    return sign | mag;
}

/* ------------------------------------------------------------------------ */
/* E4M3 (the "FN" variant): 4 exponent bits (bias 7), 3 mantissa bits,       */
/* subnormals down to 2^-9, max finite 448, 0x7F/0xFF are NaN, no inf.       */
/* [T-FMT] "Scales: Block E4M3" for NVFP4.                                   */
/* ------------------------------------------------------------------------ */
float qfo_e4m3_to_f32(uint8_t c)
{
    int s = (c >> 7) & 1, E = (c >> 3) & 15, M = c & 7;
    double v;
    if (E == 15 && M == 7) v = NAN;
    else if (E == 0) v = ldexp((double)M, -9);
    else v = ldexp(8.0 + M, E - 10);
    return (float)(s ? -v : v);
}

/* binary32 -> E4M3, round to nearest even, saturating to +-448 ("satfinite").
 * Finite inputs only. */
uint8_t qfo_e4m3_from_f32(float v)
{
    uint8_t sign = (bits_of_f32(v) >> 31) ? 0x80 : 0;
    double a = fabs((double)v);
    double r = round_to_grid(a, 3, -6);
    if (r > 448.0) r = 448.0;                                        /* satfinite */
    if (r == 0.0) return sign;
    int k; (void)frexp(r, &k);
    int e = k - 1;
    if (e < -6) return sign | (uint8_t)(r * 512.0);                  /* subnormal */
    uint8_t E = (uint8_t)(e + 7);
    uint8_t M = (uint8_t)(ldexp(r, -e) * 8.0 - 8.0);
    return sign | (uint8_t)(E << 3) | M;
}

/* ------------------------------------------------------------------------ */
/* E8M0: an 8-bit biased power of two, value 2^(code-127), 0xFF = NaN.       */
/* [T-FMT] "Scales: Block E8M0" for MXFP4.                                   */
/* Reading: the shared exponent puts the block maximum in the top binade of  */
/* E2M1 (whose largest exponent is 2): e = floor(log2(amax)) - 2, clamped to */
/* the E8M0 range [-127, 127]; an all-zero block takes e = -127.             */
/* ------------------------------------------------------------------------ */
int qfo_mx_exponent(float amax)
{
    if (!(amax > 0.0f)) return -127;
    int k;
    (void)frexp((double)amax, &k);          /* exact, subnormals included */
    int e = (k - 1) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* ------------------------------------------------------------------------ */
/* Input element types: BF16 weights/activations, or FP32 latent (master)    */
/* weights (the memory table of the project page lists the student's         */
/* trainable weights as FP32).  Every step below works on the element value.  */
/* ------------------------------------------------------------------------ */
enum { QFO_BF16 = 0, QFO_F32 = 1 };

static float xval(const void* x, int xt, int64_t i)
{
    if (xt == QFO_F32) return ((const float*)x)[i];
    return qfo_bf16_to_f32(((const uint16_t*)x)[i]);
}

static const void* xoff(const void* x, int xt, int64_t i)
{
    return xt == QFO_F32 ? (const void*)((const float*)x + i)
                         : (const void*)((const uint16_t*)x + i);
}

/* ------------------------------------------------------------------------ */
/* Tensor absolute maximum (exact: max is independent of order).             */
/* [M-NUM]: the NVFP4 tensor scale of a tie group is taken from the amax of  */
/* every tensor in the group; [M-EXP]: activation amax is tracked.           */
/* ------------------------------------------------------------------------ */
float qfo_amax_x(const void* x, int xt, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(xval(x, xt, i));
        if (a > m) m = a;
    }
    return m;
}

float qfo_amax_bf16(const uint16_t* x, int64_t n) { return qfo_amax_x(x, QFO_BF16, n); }

/* ------------------------------------------------------------------------ */
/* NVFP4 block scale derivation, one 16-element block.                       */
/* Reading (plain amax-to-largest-value scaling):                            */
/*   s_t = amax_g / (6 * 448)          FP32 tensor scale of the tie group     */
/*   sb  = E4M3( amax_b / (6 * s_t) )  block scale, RNE, saturating           */
/*   S   = f32(sb) * s_t               effective block scale                 */
/*   inv = 1 / S   (0 when S == 0)     one IEEE divide per block             */
/* With amax_g == 0 the tensor is all zeros: s_t = 0 and every sb is 0.      */
/* ------------------------------------------------------------------------ */
static void nvfp4_block_scale(float amax_b, float s_t, uint8_t* sb, float* S, float* inv)
{
    if (s_t == 0.0f) { *sb = 0; *S = 0.0f; *inv = 0.0f; return; }
    float six_st = 6.0f * s_t;
    float ratio = amax_b / six_st;
    *sb = qfo_e4m3_from_f32(ratio);
    *S = qfo_e4m3_to_f32(*sb) * s_t;
    *inv = (*S == 0.0f) ? 0.0f : 1.0f / *S;
}

/* Scaled element value q = x * inv.  When inv overflowed to +inf (S below
 * 2^-128), a zero element stays a zero of its own sign instead of 0*inf. */
static float scaled(float x, float inv)
{
    return (x == 0.0f) ? x : x * inv;
}

float qfo_nvfp4_tensor_scale(float amax_g) { return amax_g / 2688.0f; }

/* ------------------------------------------------------------------------ */
/* NVFP4 quantize-dequantize + pack of one [rows, cols] BF16 matrix whose    */
/* tie group has amax amax_g.  Blocks of 16 run along cols (the contiguous   */
/* reduction dimension).  Outputs (each may be NULL):                        */
/*   y      [rows*cols] BF16 dequantized values  y = BF16(f32(code) * S)     */
/*   codes  [rows*cols/2] bytes; element 2i in bits 0-3, 2i+1 in bits 4-7    */
/*   scales [rows*cols/16] E4M3 bytes, row-major                             */
/*   s_t    the FP32 tensor scale                                            */
/* [T-FMT] NVFP4 row; [M-NUM] tied tensor scale; [M-QDQ] quantize-dequantize.*/
/* ------------------------------------------------------------------------ */
void qfo_nvfp4_quant_x(const void* x, int xt, int64_t rows, int64_t cols, float amax_g,
                       uint16_t* y, uint8_t* codes, uint8_t* scales, float* s_t_out)
{
    float s_t = qfo_nvfp4_tensor_scale(amax_g);
    if (s_t_out) *s_t_out = s_t;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / 16; ++b) {
            const int64_t base = r * cols + b * 16;
            float amax_b = qfo_amax_x(xoff(x, xt, base), xt, 16);
            uint8_t sb; float S, inv;
            nvfp4_block_scale(amax_b, s_t, &sb, &S, &inv);
            if (scales) scales[base / 16] = sb;
            for (int i = 0; i < 16; ++i) {
                float xv = xval(x, xt, base + i);
                uint8_t c = qfo_e2m1_from_f32(scaled(xv, inv));
                if (y) y[base + i] = qfo_f32_to_bf16(qfo_e2m1_to_f32(c) * S);
                if (codes) {
                    uint8_t* p = &codes[(base + i) / 2];
                    if ((i & 1) == 0) *p = (uint8_t)((*p & 0xF0) | c);
                    else *p = (uint8_t)((*p & 0x0F) | (c << 4));
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP4 quantize-dequantize + pack.  Blocks of 32 along cols.               */
/*   e    = mx_exponent(amax_b)          (E8M0 byte = e + 127)               */
/*   code = E2M1(x * 2^-e)               (the multiply is exact)             */
/*   y    = BF16(f32(code) * 2^e)        (exact)                             */
/* Layout as NVFP4 with one E8M0 byte per 32 elements.  [T-FMT] MXFP4 row.   */
/* ------------------------------------------------------------------------ */
void qfo_mxfp4_quant_x(const void* x, int xt, int64_t rows, int64_t cols,
                       uint16_t* y, uint8_t* codes, uint8_t* scales)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / 32; ++b) {
            const int64_t base = r * cols + b * 32;
            float amax_b = qfo_amax_x(xoff(x, xt, base), xt, 32);
            int e = qfo_mx_exponent(amax_b);
            if (scales) scales[base / 32] = (uint8_t)(e + 127);
            float inv = ldexpf(1.0f, -e);
            float S = ldexpf(1.0f, e);
            for (int i = 0; i < 32; ++i) {
                float xv = xval(x, xt, base + i);
                uint8_t c = qfo_e2m1_from_f32(xv * inv);
                if (y) y[base + i] = qfo_f32_to_bf16(qfo_e2m1_to_f32(c) * S);
                if (codes) {
                    uint8_t* p = &codes[(base + i) / 2];
                    if ((i & 1) == 0) *p = (uint8_t)((*p & 0xF0) | c);
                    else *p = (uint8_t)((*p & 0x0F) | (c << 4));
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Q4_K.  [T-FMT] Q4_K row: unsigned 4-bit elements, asymmetric, 32-element  */
/* sub-blocks inside 256-element super-blocks, 6-bit sub-block scale and     */
/* min, FP16 super-block scales (d for scales, dmin for mins).               */
/* Reading (plain min/max fit):                                              */
/*  per sub-block j (32 elements):                                           */
/*    mn = min x, hi = max x                                                 */
/*    min_j   = (mn < 0) ? -mn : 0          (the stored min is subtracted)   */
/*    scale_j = (hi + min_j) / 15           (= (hi - lo) / 15, lo = min(0,mn))*/
/*  per super-block:                                                         */
/*    d    = FP16( max_j scale_j / 63 ),  dmin = FP16( max_j min_j / 63 )    */
/*    sc_j = min(RNE(scale_j / d), 63)  (0 if d == 0); m_j likewise w/ dmin   */
/*    s_j  = f32(d) * sc_j,  mm_j = f32(dmin) * m_j,  inv_j = 1/s_j (0 if 0)  */
/*  per element:                                                             */
/*    q = min(max(RNE((x + mm_j) * inv_j), 0), 15)                           */
/*    y = BF16( s_j * q - mm_j )   (a multiply, then a subtract; no FMA)     */
/* RNE(v) is the nearest integer with ties to even (nearbyint under the      */
/* default rounding mode).                                                   */
/* ------------------------------------------------------------------------ */
typedef struct {
    uint16_t d, dmin;            /* FP16 bit patterns */
    uint8_t sc[8], m[8];         /* 6-bit values */
    uint8_t q[256];              /* 4-bit values */
} q4k_super;

/* ------------------------------------------------------------------------ */
/* MSE-searched sub-block scale (the project page's "Key findings" name an   */
/* MSE-optimal quantizer as the Q4_K PTQ baseline without giving its steps;  */
/* this is a plain reading of "search the scale for least squared error").   */
/* With the sub-block's offset min_j fixed, the scale is searched over the   */
/* step counts n of the grid below -- 15 first (the min/max fit), then the   */
/* others in the listed order -- as scale = (hi + min_j) / n, and the one     */
/* with the smallest squared dequantization error                            */
/*   err = sum over i, in order, of (x_i - (scale*q_i - min_j))^2,           */
/*   q_i = clamp(RNE((x_i + min_j) * (1/scale)), 0, 15)                      */
/* is kept (a later candidate must be strictly smaller).  Everything is       */
/* binary32 with one rounding per operation.                                 */
/* ------------------------------------------------------------------------ */
static const float kQ4kSearch[9] = {15.0f, 14.0f, 14.5f, 15.5f, 16.0f, 16.5f, 17.0f, 17.5f, 18.0f};

static float q4k_sub_err(const float* v, float scale, float min_j)
{
    float inv = 1.0f / scale;
    float err = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float q = nearbyintf((v[i] + min_j) * inv);
        if (q < 0.0f) q = 0.0f;
        if (q > 15.0f) q = 15.0f;
        float deq = scale * q - min_j;
        float r = v[i] - deq;
        err = err + r * r;
    }
    return err;
}

static float q4k_search_scale(const float* v, float hi, float min_j)
{
    float range = hi + min_j;
    float best = range / kQ4kSearch[0];
    if (best == 0.0f) return best;
    float best_err = q4k_sub_err(v, best, min_j);
    for (int t = 1; t < 9; ++t) {
        float scale = range / kQ4kSearch[t];
        float err = q4k_sub_err(v, scale, min_j);
        if (err < best_err) { best_err = err; best = scale; }
    }
    return best;
}

float qfo_q4k_search_scale_one(const float* v, float hi, float min_j)
{
    return q4k_search_scale(v, hi, min_j);
}

static void q4k_fit(const void* x, int xt, int mse, q4k_super* o, uint16_t* y)
{
    float scale[8], minv[8];
    for (int j = 0; j < 8; ++j) {
        float mn = xval(x, xt, 32 * j), hi = mn;
        for (int i = 1; i < 32; ++i) {
            float v = xval(x, xt, 32 * j + i);
            if (v < mn) mn = v;
            if (v > hi) hi = v;
        }
        minv[j] = (mn < 0.0f) ? -mn : 0.0f;
        if (mse) {
            float vals[32];
            for (int i = 0; i < 32; ++i) vals[i] = xval(x, xt, 32 * j + i);
            scale[j] = q4k_search_scale(vals, hi, minv[j]);
        } else {
            scale[j] = (hi + minv[j]) / 15.0f;
        }
    }
    float max_scale = 0.0f, max_min = 0.0f;
    for (int j = 0; j < 8; ++j) {
        if (scale[j] > max_scale) max_scale = scale[j];
        if (minv[j] > max_min) max_min = minv[j];
    }
    o->d = qfo_f32_to_f16(max_scale / 63.0f);
    o->dmin = qfo_f32_to_f16(max_min / 63.0f);
    float d = qfo_f16_to_f32(o->d), dmin = qfo_f16_to_f32(o->dmin);
    for (int j = 0; j < 8; ++j) {
        float rs = (d == 0.0f) ? 0.0f : nearbyintf(scale[j] / d);
        float rm = (dmin == 0.0f) ? 0.0f : nearbyintf(minv[j] / dmin);
        o->sc[j] = (uint8_t)(rs > 63.0f ? 63.0f : rs);
        o->m[j] = (uint8_t)(rm > 63.0f ? 63.0f : rm);
        float s = d * (float)o->sc[j];
        float mm = dmin * (float)o->m[j];
        float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
        for (int i = 0; i < 32; ++i) {
            float v = (xval(x, xt, 32 * j + i) + mm) * inv;
            float q = nearbyintf(v);
            if (q < 0.0f) q = 0.0f;
            if (q > 15.0f) q = 15.0f;
            o->q[32 * j + i] = (uint8_t)q;
            if (y) {
                /* q is an unsigned integer code: dequantize from the integer */
                float sq = s * (float)o->q[32 * j + i];
                y[32 * j + i] = qfo_f32_to_bf16(sq - mm);
            }
        }
    }
}

/* The 144-byte Q4_K block, as the GGUF layout is publicly described:
 *   bytes 0-1   d (FP16), bytes 2-3 dmin (FP16)
 *   bytes 4-15  twelve bytes holding eight 6-bit scales and eight 6-bit mins:
 *                 for j < 4: scales[j]   low 6 bits = sc_j,  scales[j+4] low 6 bits = m_j
 *                 for j >= 4: scales[j+4] low nibble = sc_j & 15, high nibble = m_j & 15,
 *                             top 2 bits of scales[j-4] = sc_j >> 4,
 *                             top 2 bits of scales[j]   = m_j >> 4
 *   bytes 16-143 qs: for chunk c = 0..3 (64 elements), 32 bytes whose byte l holds
 *                element l of sub-block 2c in the low nibble and element l of
 *                sub-block 2c+1 in the high nibble.
 * This layout is written from public descriptions of the format and has not been
 * checked against the engine's own code. */
static void q4k_pack(const q4k_super* o, uint8_t* blk)
{
    blk[0] = (uint8_t)(o->d & 0xFF);    blk[1] = (uint8_t)(o->d >> 8);
    blk[2] = (uint8_t)(o->dmin & 0xFF); blk[3] = (uint8_t)(o->dmin >> 8);
    uint8_t* sc = blk + 4;
    memset(sc, 0, 12);
    for (int j = 0; j < 4; ++j) {
        sc[j] = (uint8_t)(o->sc[j] & 63);
        sc[j + 4] = (uint8_t)(o->m[j] & 63);
    }
    for (int j = 4; j < 8; ++j) {
        sc[j + 4] = (uint8_t)((o->sc[j] & 15) | ((o->m[j] & 15) << 4));
        sc[j - 4] |= (uint8_t)((o->sc[j] >> 4) << 6);
        sc[j] |= (uint8_t)((o->m[j] >> 4) << 6);
    }
    uint8_t* qs = blk + 16;
    for (int c = 0; c < 4; ++c)
        for (int l = 0; l < 32; ++l)
            qs[32 * c + l] = (uint8_t)(o->q[64 * c + l] | (o->q[64 * c + 32 + l] << 4));
}

/* Q4_K quantize-dequantize + pack of one [rows, cols] matrix, cols % 256 == 0.
 * y: [rows*cols] BF16 (may be NULL); blocks: [rows*cols/256] x 144 bytes (may be NULL). */
void qfo_q4k_quant_fit(const void* x, int xt, int mse, int64_t rows, int64_t cols,
                       uint16_t* y, uint8_t* blocks)
{
    q4k_super o;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / 256; ++b) {
            const int64_t base = r * cols + b * 256;
            q4k_fit(xoff(x, xt, base), xt, mse, &o, y ? y + base : NULL);
            if (blocks) q4k_pack(&o, blocks + (base / 256) * 144);
        }
    }
}

/* Q4_K scale/min fit of one 256-element super-block, unpacked (for pins). */
void qfo_q4k_quant_x(const void* x, int xt, int64_t rows, int64_t cols,
                     uint16_t* y, uint8_t* blocks)
{ qfo_q4k_quant_fit(x, xt, 0, rows, cols, y, blocks); }

void qfo_q4k_fit_one_fit(const void* x, int xt, int mse, uint16_t* d, uint16_t* dmin,
                         uint8_t* sc, uint8_t* m, uint8_t* q)
{
    q4k_super o;
    q4k_fit(x, xt, mse, &o, NULL);
    *d = o.d; *dmin = o.dmin;
    memcpy(sc, o.sc, 8); memcpy(m, o.m, 8); memcpy(q, o.q, 256);
}

void qfo_q4k_fit_one_x(const void* x, int xt, uint16_t* d, uint16_t* dmin, uint8_t* sc,
                       uint8_t* m, uint8_t* q)
{
    q4k_super o;
    q4k_fit(x, xt, 0, &o, NULL);
    *d = o.d; *dmin = o.dmin;
    memcpy(sc, o.sc, 8); memcpy(m, o.m, 8); memcpy(q, o.q, 256);
}

/* ------------------------------------------------------------------------ */
/* Decoders: what an engine computes from the packed bytes alone.  They are  */
/* written independently of the encoders above (they read only the packed    */
/* layout) so that decode(pack(x)) == fakequant(x) checks that the forward   */
/* pass reproduces deployment numerics [M-NUM].                              */
/* ------------------------------------------------------------------------ */
void qfo_nvfp4_decode(const uint8_t* codes, const uint8_t* scales, float s_t,
                      int64_t numel, uint16_t* y)
{
    for (int64_t i = 0; i < numel; ++i) {
        uint8_t byte = codes[i >> 1];
        uint8_t c = (i & 1) ? (byte >> 4) : (byte & 15);
        float S = qfo_e4m3_to_f32(scales[i >> 4]) * s_t;
        y[i] = qfo_f32_to_bf16(qfo_e2m1_to_f32(c) * S);
    }
}

void qfo_mxfp4_decode(const uint8_t* codes, const uint8_t* scales, int64_t numel, uint16_t* y)
{
    for (int64_t i = 0; i < numel; ++i) {
        uint8_t byte = codes[i >> 1];
        uint8_t c = (i & 1) ? (byte >> 4) : (byte & 15);
        float S = ldexpf(1.0f, (int)scales[i >> 5] - 127);
        y[i] = qfo_f32_to_bf16(qfo_e2m1_to_f32(c) * S);
    }
}

void qfo_q4k_decode(const uint8_t* blocks, int64_t numel, uint16_t* y)
{
    for (int64_t sbi = 0; sbi < numel / 256; ++sbi) {
        const uint8_t* blk = blocks + sbi * 144;
        float d = qfo_f16_to_f32((uint16_t)(blk[0] | (blk[1] << 8)));
        float dmin = qfo_f16_to_f32((uint16_t)(blk[2] | (blk[3] << 8)));
        const uint8_t* sc = blk + 4;
        const uint8_t* qs = blk + 16;
        for (int j = 0; j < 8; ++j) {
            int scj, mj;
            if (j < 4) { scj = sc[j] & 63; mj = sc[j + 4] & 63; }
            else {
                scj = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);
                mj = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
            }
            float s = d * (float)scj, mm = dmin * (float)mj;
            for (int l = 0; l < 32; ++l) {
                uint8_t byte = qs[32 * (j / 2) + l];
                int q = (j & 1) ? (byte >> 4) : (byte & 15);
                float sq = s * (float)q;
                y[sbi * 256 + 32 * j + l] = qfo_f32_to_bf16(sq - mm);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Straight-through estimator backward [M-QDQ] (Bengio et al. 2013, cited by */
/* the pages): the gradient reaches the latent weight unchanged.             */
/* mode 0: grad_x = grad_y (identity).                                       */
/* mode 1 (optional "clipped" reading): grad_x = grad_y where the element's  */
/* scaled value lies inside the representable range, +0 elsewhere:          */
/*   NVFP4 / MXFP4: |q| <= 6 with q the scaled value fed to E2M1;            */
/*   Q4_K: 0 <= (x + mm_j) * inv_j <= 15.                                    */
/* fmt: 0 NVFP4, 1 MXFP4, 2 Q4_K.  amax_g is the NVFP4 tie-group amax.       */
/* ------------------------------------------------------------------------ */
void qfo_ste_backward_x(const uint16_t* grad_y, uint16_t* grad_x, int64_t numel, int mode,
                        int fmt, const void* x, int xt, int64_t cols, float amax_g)
{
    /* fmt: 0 NVFP4, 1 MXFP4, 2 Q4_K (min/max fit), 3 Q4_K (MSE-searched fit) */
    if (mode == 0) { for (int64_t i = 0; i < numel; ++i) grad_x[i] = grad_y[i]; return; }
    int64_t rows = cols ? numel / cols : 0;
    if (fmt == 0) {
        float s_t = qfo_nvfp4_tensor_scale(amax_g);
        for (int64_t base = 0; base < rows * cols; base += 16) {
            uint8_t sb; float S, inv;
            nvfp4_block_scale(qfo_amax_x(xoff(x, xt, base), xt, 16), s_t, &sb, &S, &inv);
            for (int i = 0; i < 16; ++i) {
                float q = scaled(xval(x, xt, base + i), inv);
                grad_x[base + i] = (fabsf(q) <= 6.0f) ? grad_y[base + i] : 0;
            }
        }
    } else if (fmt == 1) {
        for (int64_t base = 0; base < rows * cols; base += 32) {
            float inv = ldexpf(1.0f, -qfo_mx_exponent(qfo_amax_x(xoff(x, xt, base), xt, 32)));
            for (int i = 0; i < 32; ++i) {
                float q = xval(x, xt, base + i) * inv;
                grad_x[base + i] = (fabsf(q) <= 6.0f) ? grad_y[base + i] : 0;
            }
        }
    } else {
        q4k_super o;
        for (int64_t base = 0; base < rows * cols; base += 256) {
            q4k_fit(xoff(x, xt, base), xt, fmt == 3, &o, NULL);
            float d = qfo_f16_to_f32(o.d), dmin = qfo_f16_to_f32(o.dmin);
            for (int j = 0; j < 8; ++j) {
                float s = d * (float)o.sc[j], mm = dmin * (float)o.m[j];
                float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
                for (int i = 0; i < 32; ++i) {
                    int64_t k = base + 32 * j + i;
                    float v = (xval(x, xt, k) + mm) * inv;
                    grad_x[k] = (v >= 0.0f && v <= 15.0f) ? grad_y[k] : 0;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* LoRA merge [M-QAD]: LoRA-QAD trains low-rank adapters on a frozen BF16    */
/* base and quantizes W + B A, not W.  Reading: the merged weight is what a  */
/* BF16 model would hold after merging --                                    */
/*   acc  = sum over k = 0..r-1, in increasing k, of B[i,k] * A[k,j]  (FP32; */
/*          each term is one fused multiply-add: acc + B*A rounded once.    */
/*          A BF16 x BF16 product has at most 16 significant bits, so this  */
/*          equals multiply-then-add unless the product underflows FP32)    */
/*   M    = BF16( W[i,j] + scale * acc )   (FP32 multiply, FP32 add, RNE)    */
/* B is [rows, r] and A is [r, cols], both BF16 row-major; scale is FP32      */
/* (alpha / r in the usual parameterisation).                                */
/* ------------------------------------------------------------------------ */
void qfo_lora_merge(const uint16_t* w, const uint16_t* b, const uint16_t* a, int64_t rows,
                    int64_t cols, int rank, float scale, uint16_t* m)
{
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t j = 0; j < cols; ++j) {
            float acc = 0.0f;
            for (int k = 0; k < rank; ++k)
                acc = fmaf(qfo_bf16_to_f32(b[i * rank + k]),
                           qfo_bf16_to_f32(a[(int64_t)k * cols + j]), acc);
            float d = scale * acc;
            m[i * cols + j] = qfo_f32_to_bf16(qfo_bf16_to_f32(w[i * cols + j]) + d);
        }
    }
}

/* BF16-input entry points (the common case). */
void qfo_nvfp4_quant(const uint16_t* x, int64_t rows, int64_t cols, float amax_g,
                     uint16_t* y, uint8_t* codes, uint8_t* scales, float* s_t_out)
{ qfo_nvfp4_quant_x(x, QFO_BF16, rows, cols, amax_g, y, codes, scales, s_t_out); }
void qfo_mxfp4_quant(const uint16_t* x, int64_t rows, int64_t cols,
                     uint16_t* y, uint8_t* codes, uint8_t* scales)
{ qfo_mxfp4_quant_x(x, QFO_BF16, rows, cols, y, codes, scales); }
void qfo_q4k_quant(const uint16_t* x, int64_t rows, int64_t cols, uint16_t* y, uint8_t* blocks)
{ qfo_q4k_quant_x(x, QFO_BF16, rows, cols, y, blocks); }
void qfo_q4k_fit_one(const uint16_t* x, uint16_t* d, uint16_t* dmin, uint8_t* sc, uint8_t* m,
                     uint8_t* q)
{ qfo_q4k_fit_one_x(x, QFO_BF16, d, dmin, sc, m, q); }
void qfo_ste_backward(const uint16_t* grad_y, uint16_t* grad_x, int64_t numel, int mode,
                      int fmt, const uint16_t* x, int64_t cols, float amax_g)
{ qfo_ste_backward_x(grad_y, grad_x, numel, mode, fmt, x, QFO_BF16, cols, amax_g); }

/* ------------------------------------------------------------------------ */
/* Array forms of the conversions, for exhaustive checks in the tests.       */
/* ------------------------------------------------------------------------ */
void qfo_e2m1_from_f32_array(const float* in, int64_t n, uint8_t* out)
{ for (int64_t i = 0; i < n; ++i) out[i] = qfo_e2m1_from_f32(in[i]); }
void qfo_e4m3_from_f32_array(const float* in, int64_t n, uint8_t* out)
{ for (int64_t i = 0; i < n; ++i) out[i] = qfo_e4m3_from_f32(in[i]); }
void qfo_f32_to_bf16_array(const float* in, int64_t n, uint16_t* out)
{ for (int64_t i = 0; i < n; ++i) out[i] = qfo_f32_to_bf16(in[i]); }
void qfo_f32_to_f16_array(const float* in, int64_t n, uint16_t* out)
{ for (int64_t i = 0; i < n; ++i) out[i] = qfo_f32_to_f16(in[i]); }

/* Scan the binary32 bit patterns [lo, hi] of one sign (lo <= hi, both with the
 * same sign bit) through a conversion and record every pattern at which the
 * result differs from the previous pattern's (the first pattern always counts).
 * which: 0 E2M1, 1 E4M3, 2 BF16, 3 FP16.  Returns the number of change points
 * (entries beyond cap are counted but not stored).  Since the bit patterns of
 * one sign are ordered by magnitude, the change list describes the whole
 * conversion over the range exactly. */
int64_t qfo_change_points(int which, uint32_t lo, uint32_t hi, uint32_t* pos,
                          uint32_t* val, int64_t cap)
{
    int64_t n = 0;
    uint32_t prev = 0xFFFFFFFFu;
    for (uint64_t u = lo; u <= hi; ++u) {
        float f = f32_of_bits((uint32_t)u);
        uint32_t r;
        switch (which) {
            case 0: r = qfo_e2m1_from_f32(f); break;
            case 1: r = qfo_e4m3_from_f32(f); break;
            case 2: r = qfo_f32_to_bf16(f); break;
            default: r = qfo_f32_to_f16(f); break;
        }
        if (r != prev) {
            if (n < cap) { pos[n] = (uint32_t)u; val[n] = r; }
            ++n;
            prev = r;
        }
    }
    return n;
}
