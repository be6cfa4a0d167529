/*
 * fp4q_ref.c -- the oracle for block-scaled FP4 quantization (MXFP4 / NVFP4)
 * and for the FOCUS fake-quant forward pass and its straight-through gradient.
 *
 * TEST INFRASTRUCTURE. This file is the plain, slow, single-threaded
 * definition of what the CUDA library must compute. Only the tests, the smoke
 * check and the CPU-baseline leg of the benchmark may load it; the product
 * path never does, and this file shares no code, header, table or constant
 * with the CUDA sources.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared.
 * On x86-64 every `float` operation below is a single IEEE-754 binary32
 * operation with round-to-nearest-even (FLT_EVAL_METHOD == 0) and nothing is
 * contracted into a fused multiply-add, so the order in which operations are
 * written here IS the arithmetic the GPU must reproduce.
 *
 * Sources (page titles; sections as they appear on each page):
 *  [FINER]  "Finer is Better (with the Right Scaling)": numerical study with
 *           OCP E2M1 data and E4M3 scale factors over block sizes 4/8/16/32
 *           (手法 1); scale strategies abs-max, prevent-zero, 4-over-6,
 *           brute force and hierarchical per-tensor + per-block scaling
 *           (手法 2); OCP E4M3 (意義と主張).
 *  [BRIDGE] "Bridging the Gap Between Promise and Performance for
 *           Microscaling FP4 Quantization": MXFP4 rounds scales to powers of
 *           two, E8M0 (技術概要 §1); blockwise Hadamard rotations of weights
 *           and activations (技術概要 §2.2 item 3; §2.1 distribution model);
 *           round-to-nearest quantization (§2.1).
 *  [FOCUS]  "FOCUS: FP4 Optimization via Coupled-Relaxation and
 *           Dual-Granularity Scaling": S_q = S_dq * c_i with c_i an FP16
 *           coefficient initialised to 1 (Metodologia §2, CRS); sub-block
 *           quantization W_k -> Q(W_k / (S_dq * c_k)) with S_dq shared by
 *           the hardware block (Metodologia §3, DGS); gradients through the
 *           non-differentiable Q by the straight-through estimator
 *           (Metodologia §1); only S_dq and the FP4 codes are deployed
 *           (Metodologia §4).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  R1  E2M1 rounding is round-to-nearest, ties to the even mantissa,
 *      saturating at +-6; the sign of the input is kept (-0.1 -> code 0x8).
 *  R2  E4M3 rounding is round-to-nearest-even, any value above 448 saturates
 *      to 448 (code 0x7E); E8M0 exponent = floor(log2 amax) - 2 clamped to
 *      [-127, 127], with amax == 0 giving -127.
 *  R3  The hierarchical FP32 global scale is s_g = amax / 2688 (= 448 * 6)
 *      for every NVFP4 strategy; s_g = 1 when that quotient is not a positive
 *      finite number (amax == 0, a non-finite or non-positive caller value).
 *  R4  Q(y / S) is computed as u = y * r with r = 1 / S (one division per
 *      block and candidate); if r overflows it is replaced by the largest
 *      finite float of the same sign. A zero scale S == 0 encodes every
 *      element of the block as code 0x0 with dequantized value +0.
 *  R5  Blockwise Hadamard: Sylvester order, stages h = 1, 2, 4, ... ascending,
 *      then one multiply by k_n, the float nearest 1/sqrt(n). Rotated values
 *      stay fp32; dequantized values and MSE are in the rotated domain.
 *  R6  Sums over a block use the adjacent-pair tree: for h = 1, 2, ..., B/2,
 *      v[i] += v[i + h] for i = 0, 2h, 4h, ...; MSE = SSE / B.
 *  R7  4-over-6 keeps target 4 only if SSE_4 < SSE_6 (a tie keeps 6); brute
 *      force scans codes 0x01..0x7E upward and keeps a strictly smaller SSE
 *      (a tie keeps the lower code); prevent-zero = max(abs-max code, 0x01).
 *  R8  Packed codes: byte j holds element 2j in its low nibble and element
 *      2j+1 in its high nibble. Scales are one byte per block, row-major.
 *  R9  FOCUS backward: dQ/du := 1 everywhere (no clipping), S_dq receives no
 *      gradient, dc_k = -(tsum_k(g * W) / (c_k * c_k)); the CRS per-block c_i
 *      is the special case sub-block == block.
 *  R13 Dequantization back to the original domain applies the normalised
 *      rotation again (same stages and k_n): H_n is symmetric and
 *      H_n H_n = n I, so it is its own inverse up to the rounding of k_n.
 *  R11 MXFP4 "brute force" is the MSE-optimised grid of [BRIDGE] 技術概要
 *      §2.2 item 1 (per group, the scale minimising the MSE) over the
 *      format's own scales: every E8M0 byte 0..254, scanned upward, a strictly
 *      smaller SSE wins, a tie keeps the lower byte.
 *  R17 UE5M3 block scales ([FINER] 意義と主張 names the unsigned wide-exponent
 *      format without its encoding): 8 bits, 5 exponent bits with the IEEE
 *      bias 15, 3 mantissa bits, exponent field 0 subnormal (m * 2^-17),
 *      only 0xFF NaN as in OCP E4M3; largest 1.75 * 2^16 (0xFE). Its range
 *      needs no hierarchical scaling, so s_g = 1: candidate code =
 *      RNE_UE5M3_sat(amax / T); the four strategies as for E4M3, brute force
 *      over codes 0x01..0xFE.
 *  R18 MR-GPTQ ([BRIDGE] 技術概要 §2.2 lists its parts without formulas):
 *      GPTQ error feedback over the upper Cholesky factor U of the inverse
 *      (damped) Hessian, with static groups -- block scales fixed beforehand
 *      from the original weights by any scale strategy (the MSE-optimised
 *      grid is the brute force / MSE grid) -- and static activation
 *      reordering as a processing order of the columns (codes stay in the
 *      original order). Lazy batch updates over 128 positions; within a
 *      batch each update is one fma, the trailing update one fma-chain sum
 *      per element followed by one subtraction. The rotation part is not
 *      in this step: it takes the bf16 weights as stored.
 *  R15 FOCUS calibration: the pages learn c by gradient descent through the
 *      STE but name neither the optimizer nor the precision of the update.
 *      The learnable state is an fp32 master copy of c; the forward uses its
 *      fp16 rounding (the pages' FP16 parameter) and the gradient of R9 is
 *      taken at that fp16 value. Optimizers: plain SGD, and Adam in the
 *      efficient ordering Kingma & Ba give beside their algorithm: the step
 *      size alpha_t = lr sqrt(1 - b2^t) / (1 - b1^t) is computed in double
 *      and rounded once to fp32, and eps is added to sqrt(v).
 *  R16 The fused calibration step minimises the weight-reconstruction loss
 *      sum (W_hat - W)^2 with g = 2 (W_hat - W) in fp32. (At c == 1 every
 *      element already lands on its nearest point of the S_dq grid, so this
 *      loss cannot go lower; losses that couple elements, such as a layer's
 *      output, are served by the update from an external gradient.)
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define REF_FMT_NVFP4 0
#define REF_FMT_MXFP4 1
#define REF_FMT_UE5M3 2

#define REF_ABSMAX 0
#define REF_PREVENT_ZERO 1
#define REF_FOUR_OVER_SIX 2
#define REF_BRUTE_FORCE 3

#define REF_OK 0
#define REF_ERR_ARG 1

/* ------------------------------------------------------------------------ */
/* Number formats, by their definitions.                                     */
/* ------------------------------------------------------------------------ */

/* OCP E2M1 magnitude of the 3 low bits m of a code: 2 exponent bits (bias 1)
 * and 1 mantissa bit; exponent field 0 is subnormal. [FINER] 手法 1 names the
 * format; its 4-over-6 bullet names 4.0 and 6.0 as the two largest values. */
double ref_e2m1_magnitude(int m)
{
    int e = (m >> 1) & 3;
    int f = m & 1;
    if (e == 0)
        return 0.5 * f;
    return ldexp(1.0 + 0.5 * f, e - 1);
}

/* Signed value of a 4-bit E2M1 code (bit 3 is the sign). */
double ref_e2m1_value(int code)
{
    double v = ref_e2m1_magnitude(code & 7);
    return (code & 8) ? -v : v;
}

/* OCP E4M3 value of a byte 0..0x7E (non-negative codes): 4 exponent bits with
 * bias 7, 3 mantissa bits, exponent field 0 subnormal; 0x7F is NaN.
 * [FINER] 意義と主張 (OCP E4M3); 手法 2 (E4M3 scale factors). */
double ref_e4m3_value(int code)
{
    int e = (code >> 3) & 15;
    int m = code & 7;
    if ((code & 0x7F) == 0x7F)
        return NAN;
    double v = (e == 0) ? ldexp(m / 8.0, 1 - 7) : ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -v : v;
}

/* E8M0 value of a byte: a bare power of two 2^(b - 127); 255 is NaN.
 * [BRIDGE] 技術概要 §1 (MXFP4 scales are powers of two, E8M0). */
double ref_e8m0_value(int b)
{
    if (b == 255)
        return NAN;
    return ldexp(1.0, b - 127);
}

/* bf16 bits -> float: a bf16 number is the upper half of a binary32. */
float ref_bf16_to_float(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, 4);
    return f;
}

/* IEEE binary16 bits -> float, by the format definition (bias 15). */
float ref_fp16_to_float(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1024.0 + m, e - 25);
    return (float)(s ? -v : v);
}

static uint32_t f2bits(float f)
{
    uint32_t b;
    memcpy(&b, &f, 4);
    return b;
}

static float bits2f(uint32_t b)
{
    float f;
    memcpy(&f, &b, 4);
    return f;
}

/* float -> bf16 bits, round to nearest, ties to even (finite inputs). The two
 * candidates are the bf16 numbers just below and just above |v| in magnitude;
 * a value past the largest finite bf16 rounds as if 2^128 were the next
 * number, and then becomes infinity, as IEEE rounding does. */
uint16_t ref_float_to_bf16(float v)
{
    uint32_t b = f2bits(v);
    uint32_t sign = b & 0x80000000u;
    uint32_t mag = b & 0x7FFFFFFFu;
    if (mag > 0x7F800000u)
        return (uint16_t)((b >> 16) | 0x40); /* NaN stays NaN */
    if (mag == 0x7F800000u)
        return (uint16_t)(b >> 16); /* +-infinity */
    uint32_t lo = mag & 0xFFFF0000u;
    uint32_t hi = lo + 0x10000u;
    double x = (double)bits2f(mag);
    double vlo = (double)bits2f(lo);
    double vhi = (hi >= 0x7F800000u) ? ldexp(1.0, 128) : (double)bits2f(hi);
    double dlo = x - vlo, dhi = vhi - x;
    uint32_t pick;
    if (dlo < dhi)
        pick = lo;
    else if (dhi < dlo)
        pick = hi;
    else
        pick = ((lo >> 16) & 1) ? hi : lo;
    if (pick >= 0x7F800000u)
        pick = 0x7F800000u;
    return (uint16_t)((sign | pick) >> 16);
}

/* ------------------------------------------------------------------------ */
/* Rounding to the formats (readings R1, R2).                                */
/* ------------------------------------------------------------------------ */

/* Round u to the nearest E2M1 value, ties to the even mantissa index m,
 * saturating at 6; the sign bit of u is kept. Returns the 4-bit code. */
int ref_rne_e2m1(float u)
{
    double a = fabs((double)u);
    int sign = signbit(u) ? 8 : 0;
    int best = 7;
    if (a < 6.0) {
        best = 0;
        for (int m = 1; m < 8; m++) {
            double dm = fabs(a - ref_e2m1_magnitude(m));
            double db = fabs(a - ref_e2m1_magnitude(best));
            if (dm < db || (dm == db && (m & 1) == 0))
                best = m;
        }
    }
    return sign | best;
}

/* Round v >= 0 to the nearest non-negative finite E4M3 value, ties to the
 * even code, saturating above 448 (code 0x7E). The codes 0..0x7E increase
 * with their value, so the two neighbours of v are found by bisection over
 * that enumerated table. */
int ref_rne_e4m3_sat(float v)
{
    if (!(v <= 448.0f))
        return 0x7E;
    double x = (double)v;
    if (x <= ref_e4m3_value(0))
        return 0;
    /* smallest k in 1..0x7E with value(k) >= x; it exists since x <= 448 */
    int lo = 0, hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi) / 2;
        if (ref_e4m3_value(mid) >= x)
            hi = mid;
        else
            lo = mid + 1;
    }
    int k = lo;
    if (ref_e4m3_value(k) == x)
        return k;
    double dk = ref_e4m3_value(k) - x;
    double dp = x - ref_e4m3_value(k - 1);
    if (dp < dk)
        return k - 1;
    if (dk < dp)
        return k;
    return (k & 1) ? k - 1 : k;
}

/* UE5M3 value of a byte 0..0xFE (reading R17): unsigned, 5 exponent bits with
 * bias 15, 3 mantissa bits, exponent field 0 subnormal; 0xFF is NaN.
 * [FINER] 意義と主張 (UE5M3 as the wide-range scale format compared with
 * E4M3 + hierarchical scaling). */
double ref_ue5m3_value(int code)
{
    int e = (code >> 3) & 31;
    int m = code & 7;
    if ((code & 0xFF) == 0xFF)
        return NAN;
    return (e == 0) ? ldexp(m / 8.0, 1 - 15) : ldexp(1.0 + m / 8.0, e - 15);
}

/* Round v >= 0 to the nearest finite UE5M3 value, ties to the even code,
 * saturating above the largest value 1.75 * 2^16 (code 0xFE); bisection over
 * the enumerated codes 0..0xFE, which increase with their value. */
int ref_rne_ue5m3_sat(float v)
{
    double top = ref_ue5m3_value(0xFE);
    if (!((double)v <= top))
        return 0xFE;
    double x = (double)v;
    if (x <= 0.0)
        return 0;
    int lo = 0, hi = 0xFE;
    while (lo < hi) {
        int mid = (lo + hi) / 2;
        if (ref_ue5m3_value(mid) >= x)
            hi = mid;
        else
            lo = mid + 1;
    }
    int k = lo;
    if (ref_ue5m3_value(k) == x)
        return k;
    double dk = ref_ue5m3_value(k) - x;
    double dp = x - ref_ue5m3_value(k - 1);
    if (dp < dk)
        return k - 1;
    if (dk < dp)
        return k;
    return (k & 1) ? k - 1 : k;
}

/* E8M0 exponent for a block abs-max a >= 0: floor(log2 a) - 2, clamped to
 * [-127, 127]; a == 0 gives -127. frexp writes a = f * 2^k, f in [0.5, 1),
 * so floor(log2 a) = k - 1 exactly. */
int ref_e8m0_exponent(float a)
{
    if (a == 0.0f)
        return -127;
    int k;
    (void)frexp((double)a, &k);
    int e = (k - 1) - 2;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* ------------------------------------------------------------------------ */
/* Reductions and the Hadamard rotation (readings R5, R6).                   */
/* ------------------------------------------------------------------------ */

/* Adjacent-pair tree sum of v[0..n), n a power of two; v is overwritten. */
float ref_tsum(float* v, int n)
{
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i + h < n; i += 2 * h)
            v[i] = v[i] + v[i + h];
    return v[0];
}

/* The float nearest 1/sqrt(n) for the supported rotation sizes. */
float ref_hadamard_k(int n)
{
    switch (n) {
    case 16: return bits2f(0x3e800000u);  /* 0.25 */
    case 32: return bits2f(0x3e3504f3u);  /* 0.17677669... */
    case 64: return bits2f(0x3e000000u);  /* 0.125 */
    case 128: return bits2f(0x3db504f3u); /* 0.08838834... */
    default: return NAN;
    }
}

/* In-place normalised fast Walsh-Hadamard transform of t[0..n):
 * stages h = 1, 2, 4, ..., n/2 with (t[i], t[i+h]) <- (t[i]+t[i+h], t[i]-t[i+h])
 * for every i with (i & h) == 0, then t[i] <- t[i] * k_n. This is y = H_n t / sqrt(n)
 * with the Sylvester matrix H_2m = [[H_m, H_m], [H_m, -H_m]].
 * [BRIDGE] 技術概要 §2.2 item 3 (blockwise rotations), §2.1. */
void ref_fwht(float* t, int n)
{
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; i++)
            if ((i & h) == 0) {
                float a = t[i], b = t[i + h];
                t[i] = a + b;
                t[i + h] = a - b;
            }
    float k = ref_hadamard_k(n);
    for (int i = 0; i < n; i++)
        t[i] = t[i] * k;
}

/* Widen one row of bf16 to float and rotate it chunk by chunk (rot == 0: no
 * rotation). */
static void load_row(const uint16_t* x, int64_t cols, int rot, float* y)
{
    for (int64_t j = 0; j < cols; j++)
        y[j] = ref_bf16_to_float(x[j]);
    if (rot > 0)
        for (int64_t j = 0; j < cols; j += rot)
            ref_fwht(y + j, rot);
}

/* Tensor abs-max of the (rotated) tensor: the input of the FP32 global scale
 * of hierarchical scaling, [FINER] 手法 2. */
float ref_global_amax(const uint16_t* x, int64_t rows, int64_t cols, int rot)
{
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    float g = 0.0f;
    for (int64_t i = 0; i < rows; i++) {
        load_row(x + i * cols, cols, rot, y);
        for (int64_t j = 0; j < cols; j++) {
            float a = fabsf(y[j]);
            if (a > g)
                g = a;
        }
    }
    free(y);
    return g;
}

/* s_g from the tensor abs-max (reading R3). */
float ref_global_scale(float g)
{
    float sg = g / 2688.0f;
    if (!(sg > 0.0f) || !(g <= FLT_MAX))
        sg = 1.0f;
    return sg;
}

/* ------------------------------------------------------------------------ */
/* One block (readings R4, R6).                                              */
/* ------------------------------------------------------------------------ */

/* r = 1 / S with the overflow guard of R4. */
static float guarded_reciprocal(float S)
{
    float r = 1.0f / S;
    if (isinf(r))
        r = signbit(r) ? -FLT_MAX : FLT_MAX;
    return r;
}

/* Quantize y[0..B) with dequantization scale S: q = RNE_E2M1(y * (1/S)),
 * yhat = value(q) * S; returns the block's sum of squared errors. */
static float quant_block(const float* y, int B, float S, uint8_t* q, float* yhat)
{
    float e[128];
    if (S == 0.0f) {
        for (int i = 0; i < B; i++) {
            q[i] = 0;
            yhat[i] = 0.0f;
            float d = y[i] - yhat[i];
            e[i] = d * d;
        }
    } else {
        float r = guarded_reciprocal(S);
        for (int i = 0; i < B; i++) {
            float u = y[i] * r;
            q[i] = (uint8_t)ref_rne_e2m1(u);
            yhat[i] = (float)ref_e2m1_value(q[i]) * S;
            float d = y[i] - yhat[i];
            e[i] = d * d;
        }
    }
    return ref_tsum(e, B);
}

/* The block-scale formats of the NVFP4 family: E4M3 (under the FP32 global
 * scale s_g) and UE5M3 (reading R17: its range needs no global scale, so s_g
 * is 1). max_code is the largest finite code. */
typedef struct {
    int (*rne)(float);
    double (*value)(int);
    int max_code;
} scale_format;

static const scale_format FMT_E4M3 = {ref_rne_e4m3_sat, ref_e4m3_value, 0x7E};
static const scale_format FMT_UE5M3 = {ref_rne_ue5m3_sat, ref_ue5m3_value, 0xFE};

/* Scale candidate for target T (6 = abs-max, 4 = the 4-over-6 alternative):
 * raw = amax / (T * s_g), code = RNE_sat(raw) in the scale format,
 * S = value(code) * s_g. [FINER] 手法 2 (abs-max rounded to the nearest E4M3
 * value; 4-over-6 targets; hierarchical scaling). */
static int nv_candidate(float amax, float T, float sg, float* S)
{
    float den = T * sg;
    float raw = amax / den;
    int c = ref_rne_e4m3_sat(raw);
    *S = (float)ref_e4m3_value(c) * sg;
    return c;
}

static int scale_candidate(const scale_format* f, float amax, float T, float sg, float* S)
{
    float den = T * sg;
    float raw = amax / den;
    int c = f->rne(raw);
    *S = (float)f->value(c) * sg;
    return c;
}

/* Selects the block scale (E4M3 or UE5M3 format f) of one block by the given
 * strategy and quantizes it with that scale. Returns the block SSE; writes
 * scale byte, codes, yhat. */
static float nv_block(const float* y, int B, int strat, float sg, const scale_format* f,
                      uint8_t* scale, uint8_t* q, float* yhat)
{
    float amax = 0.0f;
    for (int i = 0; i < B; i++) {
        float a = fabsf(y[i]);
        if (a > amax)
            amax = a;
    }
    float S6;
    int c6 = scale_candidate(f, amax, 6.0f, sg, &S6);
    if (strat == REF_ABSMAX) {
        *scale = (uint8_t)c6;
        return quant_block(y, B, S6, q, yhat);
    }
    if (strat == REF_PREVENT_ZERO) {
        /* clip the scale to the smallest positive value of the format (code
         * 0x01: 2^-9 in E4M3), [FINER] 手法 2 prevent-zero */
        int c = c6 < 1 ? 1 : c6;
        float S = (float)f->value(c) * sg;
        *scale = (uint8_t)c;
        return quant_block(y, B, S, q, yhat);
    }
    if (strat == REF_FOUR_OVER_SIX) {
        uint8_t q4[128];
        float yh4[128];
        float S4;
        int c4 = scale_candidate(f, amax, 4.0f, sg, &S4);
        float sse6 = quant_block(y, B, S6, q, yhat);
        float sse4 = quant_block(y, B, S4, q4, yh4);
        if (sse4 < sse6) {
            memcpy(q, q4, (size_t)B);
            memcpy(yhat, yh4, sizeof(float) * (size_t)B);
            *scale = (uint8_t)c4;
            return sse4;
        }
        *scale = (uint8_t)c6;
        return sse6;
    }
    /* brute force over every positive finite code, [FINER] 手法 2 */
    uint8_t qt[128];
    float yht[128];
    int best_c = -1;
    float best = 0.0f;
    for (int c = 0x01; c <= f->max_code; c++) {
        float S = (float)f->value(c) * sg;
        float sse = quant_block(y, B, S, qt, yht);
        if (best_c < 0 || sse < best) {
            best = sse;
            best_c = c;
        }
    }
    float S = (float)f->value(best_c) * sg;
    *scale = (uint8_t)best_c;
    return quant_block(y, B, S, q, yhat);
}

/* MXFP4 block. abs-max: S = 2^e with e the E8M0 exponent of the block
 * abs-max ([BRIDGE] 技術概要 §1). brute force (reading R11): the
 * MSE-optimised grid of [BRIDGE] 技術概要 §2.2 item 1 restricted to the
 * format's own scales -- every E8M0 byte 0..254 (S = 2^(byte - 127)) scanned
 * upward, a strictly smaller SSE wins (a tie keeps the lower byte). */
static float mx_block(const float* y, int B, int strat, uint8_t* scale, uint8_t* q, float* yhat)
{
    if (strat == REF_BRUTE_FORCE) {
        uint8_t qt[128];
        float yht[128];
        int best_b = -1;
        float best = 0.0f;
        for (int b = 0; b <= 254; b++) {
            float sse = quant_block(y, B, (float)ref_e8m0_value(b), qt, yht);
            if (best_b < 0 || sse < best) {
                best = sse;
                best_b = b;
            }
        }
        *scale = (uint8_t)best_b;
        return quant_block(y, B, (float)ref_e8m0_value(best_b), q, yhat);
    }
    float amax = 0.0f;
    for (int i = 0; i < B; i++) {
        float a = fabsf(y[i]);
        if (a > amax)
            amax = a;
    }
    int e = ref_e8m0_exponent(amax);
    *scale = (uint8_t)(e + 127);
    float S = (float)ldexp(1.0, e);
    return quant_block(y, B, S, q, yhat);
}

static int valid_common(int64_t rows, int64_t cols, int fmt, int block, int rot)
{
    if (rows <= 0 || cols <= 0)
        return 0;
    if (fmt == REF_FMT_MXFP4 && block != 32)
        return 0;
    if (fmt != REF_FMT_MXFP4 && block != 4 && block != 8 && block != 16 && block != 32)
        return 0;
    if (fmt != REF_FMT_NVFP4 && fmt != REF_FMT_MXFP4 && fmt != REF_FMT_UE5M3)
        return 0;
    if (rot != 0 && rot != 16 && rot != 32 && rot != 64 && rot != 128)
        return 0;
    if (cols % block != 0 || (rot > 0 && cols % rot != 0))
        return 0;
    return 1;
}

/* ------------------------------------------------------------------------ */
/* Whole-tensor entry points.                                                */
/* ------------------------------------------------------------------------ */

/* Quantize a bf16 [rows, cols] tensor (blocks along cols).
 * global_amax_in: NVFP4 only, NULL to compute it over the rotated tensor.
 * global_scale_out: NVFP4 only, receives s_g (may be NULL).
 * codes: [rows, cols/2] packed (R8); scales: [rows, cols/block];
 * block_mse, dq_f32, dq_bf16: optional (NULL to skip). */
int ref_quantize(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int block, int strat,
                 int rot, const float* global_amax_in, float* global_scale_out, uint8_t* codes,
                 uint8_t* scales, float* block_mse, float* dq_f32, uint16_t* dq_bf16)
{
    if (!valid_common(rows, cols, fmt, block, rot))
        return REF_ERR_ARG;
    if (fmt == REF_FMT_MXFP4 && strat != REF_ABSMAX && strat != REF_BRUTE_FORCE)
        return REF_ERR_ARG;
    if (strat < REF_ABSMAX || strat > REF_BRUTE_FORCE)
        return REF_ERR_ARG;
    float sg = 1.0f;
    if (fmt == REF_FMT_NVFP4) {
        float g = global_amax_in ? *global_amax_in : ref_global_amax(x, rows, cols, rot);
        sg = ref_global_scale(g);
        if (global_scale_out)
            *global_scale_out = sg;
    }
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    uint8_t q[128];
    float yhat[128];
    int64_t nb = cols / block;
    for (int64_t i = 0; i < rows; i++) {
        load_row(x + i * cols, cols, rot, y);
        for (int64_t b = 0; b < nb; b++) {
            const float* yb = y + b * block;
            uint8_t sc;
            float sse = (fmt == REF_FMT_MXFP4)
                            ? mx_block(yb, block, strat, &sc, q, yhat)
                            : nv_block(yb, block, strat, sg,
                                       fmt == REF_FMT_UE5M3 ? &FMT_UE5M3 : &FMT_E4M3, &sc, q, yhat);
            int64_t base = i * cols + b * block;
            scales[i * nb + b] = sc;
            if (block_mse)
                block_mse[i * nb + b] = sse / (float)block;
            for (int j = 0; j < block; j += 2)
                codes[(base + j) / 2] = (uint8_t)(q[j] | (q[j + 1] << 4));
            for (int j = 0; j < block; j++) {
                if (dq_f32)
                    dq_f32[base + j] = yhat[j];
                if (dq_bf16)
                    dq_bf16[base + j] = ref_float_to_bf16(yhat[j]);
            }
        }
    }
    free(y);
    return REF_OK;
}

/* Dequantization scale of one block from its stored byte. */
static float block_scale(int fmt, uint8_t sc, float sg)
{
    if (fmt == REF_FMT_MXFP4)
        return (float)ref_e8m0_value(sc);
    if (fmt == REF_FMT_UE5M3)
        return (float)ref_ue5m3_value(sc);
    return (float)ref_e4m3_value(sc) * sg;
}

/* Dequantize packed codes: yhat = value(q) * S. global_scale: s_g (NVFP4). */
int ref_dequantize(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                   int64_t rows, int64_t cols, int fmt, int block, float* out_f32,
                   uint16_t* out_bf16)
{
    if (!valid_common(rows, cols, fmt, block, 0))
        return REF_ERR_ARG;
    float sg = (fmt == REF_FMT_NVFP4) ? *global_scale : 1.0f;
    for (int64_t k = 0; k < rows * cols; k++) {
        uint8_t byte = codes[k / 2];
        int q = (k & 1) ? (byte >> 4) : (byte & 15);
        float S = block_scale(fmt, scales[k / block], sg);
        float v = (float)ref_e2m1_value(q) * S;
        if (out_f32)
            out_f32[k] = v;
        if (out_bf16)
            out_bf16[k] = ref_float_to_bf16(v);
    }
    return REF_OK;
}

/* Dequantize, then return to the original domain: yhat = value(q) * S as in
 * ref_dequantize, then every rot-wide chunk of a row through the normalised
 * transform once more (reading R13: the Sylvester H_n is symmetric with
 * H_n H_n = n I, so the normalised rotation is its own inverse, exactly for
 * n = 16 and 64 where k_n^2 n = 1, up to the rounding of k_n otherwise).
 * [BRIDGE] 技術概要 §2.2 item 3 (blockwise rotations). rot == 0 is plain
 * dequantization. */
int ref_dequantize_unrotate(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                            int64_t rows, int64_t cols, int fmt, int block, int rot,
                            float* out_f32, uint16_t* out_bf16)
{
    if (!valid_common(rows, cols, fmt, block, rot))
        return REF_ERR_ARG;
    float sg = (fmt == REF_FMT_NVFP4) ? *global_scale : 1.0f;
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    for (int64_t i = 0; i < rows; i++) {
        for (int64_t j = 0; j < cols; j++) {
            int64_t k = i * cols + j;
            uint8_t byte = codes[k / 2];
            int q = (k & 1) ? (byte >> 4) : (byte & 15);
            y[j] = (float)ref_e2m1_value(q) * block_scale(fmt, scales[k / block], sg);
        }
        if (rot > 0)
            for (int64_t j = 0; j < cols; j += rot)
                ref_fwht(y + j, rot);
        for (int64_t j = 0; j < cols; j++) {
            if (out_f32)
                out_f32[i * cols + j] = y[j];
            if (out_bf16)
                out_bf16[i * cols + j] = ref_float_to_bf16(y[j]);
        }
    }
    free(y);
    return REF_OK;
}

/* The product of two quantized operands, as the FP4 matrix multiplication of
 * [BRIDGE] 技術概要 §2.3 computes it: D[m][n] = s_a * s_b * sum_k A[m][k] B[n][k]
 * with A [M, K] and B [N, K] given by their packed codes and row-major block
 * scales (R8), A[m][k] = value(code) * block scale (E4M3 for NVFP4, E8M0 for
 * MXFP4) and s_a, s_b the NVFP4 global scales (1 for MXFP4). Accumulated in
 * double, rounded once to float. */
int ref_fp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, float a_sg, const uint8_t* b_codes,
                 const uint8_t* b_scales, float b_sg, int64_t M, int64_t N, int64_t K, int fmt,
                 float* d)
{
    int block = (fmt == REF_FMT_MXFP4) ? 32 : 16;
    if (M <= 0 || N <= 0 || K <= 0 || K % block != 0 || (fmt != REF_FMT_NVFP4 && fmt != REF_FMT_MXFP4))
        return REF_ERR_ARG;
    double alpha = (fmt == REF_FMT_NVFP4) ? (double)a_sg * (double)b_sg : 1.0;
    double* av = (double*)malloc(sizeof(double) * (size_t)K);
    double* bv = (double*)malloc(sizeof(double) * (size_t)(N * K));
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            int64_t t = n * K + k;
            int q = (k & 1) ? (b_codes[t / 2] >> 4) : (b_codes[t / 2] & 15);
            bv[t] = ref_e2m1_value(q) * block_scale(fmt, b_scales[n * (K / block) + k / block], 1.0f);
        }
    for (int64_t m = 0; m < M; m++) {
        for (int64_t k = 0; k < K; k++) {
            int64_t t = m * K + k;
            int q = (k & 1) ? (a_codes[t / 2] >> 4) : (a_codes[t / 2] & 15);
            av[k] = ref_e2m1_value(q) * block_scale(fmt, a_scales[m * (K / block) + k / block], 1.0f);
        }
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += av[k] * bv[n * K + k];
            d[m * N + n] = (float)(alpha * acc);
        }
    }
    free(av);
    free(bv);
    return REF_OK;
}

/* GPTQ error feedback with static groups ([BRIDGE] 技術概要 §2.2: MR-GPTQ =
 * GPTQ with the MSE-optimised grid, static activation reordering and
 * rotations), reading R18. The block scales are fixed beforehand (static
 * groups: scales[rows, K/block] from ref_quantize of the original weights,
 * any strategy; s_g for NVFP4). The columns are processed in the order perm
 * (processing position j -> original column perm[j]; NULL = identity) with U
 * the upper Cholesky factor of the inverse Hessian in that order (fp32
 * [K, K] row-major). Per row, in blocks of 128 positions (K % 128 == 0):
 *   for each position j of the block: S = scale of the block holding column
 *     perm[j]; q = RNE_E2M1(w_j * (1/S)) (code 0 if S == 0); the error
 *     e_j = (w_j - value(q) * S) / U[j][j]; the later positions k of the
 *     block take w_k = fma(-e_j, U[j][k], w_k), j ascending;
 *   then every position k after the block: t = fma sum of e_j * U[j][k] over
 *     the block's j ascending from t = 0, and w_k = w_k - t.
 * Codes are written at the original column (packed as in R8). Rows are
 * independent.
 * rot > 0: the rotation of MR-GPTQ comes first -- each row is rotated chunk by
 * chunk (rot-wide blockwise Hadamard of the original column order, exactly
 * the quantizer's rotation, load_row) and the error feedback runs on the
 * rotated fp32 weights; scales, U and perm then belong to the rotated basis
 * (static scales from ref_quantize with the same rot; U from the Hessian of
 * the rotated inputs). The codes are those of the rotated weights. */
int ref_gptq(const uint16_t* w, int64_t rows, int64_t K, int fmt, int block, int rot,
             const uint8_t* scales, float sg, const float* U, const int32_t* perm,
             uint8_t* codes)
{
    if (!valid_common(rows, K, fmt, block, rot) || K % 128 != 0)
        return REF_ERR_ARG;
    if (perm) {
        uint8_t* seen = (uint8_t*)calloc((size_t)K, 1);
        int ok = 1;
        for (int64_t j = 0; j < K && ok; j++) {
            if (perm[j] < 0 || perm[j] >= K || seen[perm[j]])
                ok = 0;
            else
                seen[perm[j]] = 1;
        }
        free(seen);
        if (!ok)
            return REF_ERR_ARG;
    }
    float* W = (float*)malloc(sizeof(float) * (size_t)K);
    float* Y = (float*)malloc(sizeof(float) * (size_t)K);
    float E[128];
    int64_t nb = K / block;
    memset(codes, 0, (size_t)(rows * K / 2));
    for (int64_t i = 0; i < rows; i++) {
        load_row(w + i * K, K, rot, Y);
        for (int64_t j = 0; j < K; j++)
            W[j] = Y[perm ? perm[j] : j];
        for (int64_t b0 = 0; b0 < K; b0 += 128) {
            for (int jj = 0; jj < 128; jj++) {
                int64_t j = b0 + jj;
                int64_t col = perm ? perm[j] : j;
                float S = block_scale(fmt, scales[i * nb + col / block], sg);
                int q = 0;
                float deq = 0.0f;
                if (S != 0.0f) {
                    float u = W[j] * guarded_reciprocal(S);
                    q = ref_rne_e2m1(u);
                    deq = (float)ref_e2m1_value(q) * S;
                }
                float d = W[j] - deq;
                E[jj] = d / U[j * K + j];
                int64_t t = i * K + col;
                codes[t / 2] = (uint8_t)(codes[t / 2] | (q << (4 * (t & 1))));
                for (int kk = jj + 1; kk < 128; kk++)
                    W[b0 + kk] = fmaf(-E[jj], U[j * K + b0 + kk], W[b0 + kk]);
            }
            for (int64_t k = b0 + 128; k < K; k++) {
                float t = 0.0f;
                for (int jj = 0; jj < 128; jj++)
                    t = fmaf(E[jj], U[(b0 + jj) * K + k], t);
                W[k] = W[k] - t;
            }
        }
    }
    free(W);
    free(Y);
    return REF_OK;
}

/* Per-block MSE of the rotated x against dequantize(codes, scales). */
int ref_block_mse(const uint16_t* x, const uint8_t* codes, const uint8_t* scales,
                  const float* global_scale, int64_t rows, int64_t cols, int fmt, int block,
                  int rot, float* block_mse)
{
    if (!valid_common(rows, cols, fmt, block, rot))
        return REF_ERR_ARG;
    float sg = (fmt == REF_FMT_NVFP4) ? *global_scale : 1.0f;
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    float e[128];
    int64_t nb = cols / block;
    for (int64_t i = 0; i < rows; i++) {
        load_row(x + i * cols, cols, rot, y);
        for (int64_t b = 0; b < nb; b++) {
            float S = block_scale(fmt, scales[i * nb + b], sg);
            for (int j = 0; j < block; j++) {
                int64_t k = i * cols + b * block + j;
                uint8_t byte = codes[k / 2];
                int q = (k & 1) ? (byte >> 4) : (byte & 15);
                float yhat = (float)ref_e2m1_value(q) * S;
                float d = y[b * block + j] - yhat;
                e[j] = d * d;
            }
            block_mse[i * nb + b] = ref_tsum(e, block) / (float)block;
        }
    }
    free(y);
    return REF_OK;
}

/* FOCUS forward (CRS + DGS): per hardware block the dequantization scale S_dq
 * is the format's abs-max scale; per sub-block k of `sub` elements,
 * W_hat = S_dq * Q(W / (S_dq * c_k)). c: fp16 bits [rows, cols/sub].
 * [FOCUS] Metodologia §2 (S_q = S_dq * c_i), §3 (sub-block formula), §4. */
int ref_focus_fwd(const uint16_t* w, const uint16_t* c, int64_t rows, int64_t cols, int fmt,
                  int block, int sub, const float* global_amax_in, float* global_scale_out,
                  float* w_hat_f32, uint16_t* w_hat_bf16, uint8_t* codes, uint8_t* scales)
{
    if (!valid_common(rows, cols, fmt, block, 0))
        return REF_ERR_ARG;
    if (fmt == REF_FMT_UE5M3)
        return REF_ERR_ARG; /* FOCUS is defined for MXFP4 and NVFP4 */
    if (sub < 1 || block % sub != 0 || (sub & (sub - 1)) != 0)
        return REF_ERR_ARG;
    float sg = 1.0f;
    if (fmt == REF_FMT_NVFP4) {
        float g = global_amax_in ? *global_amax_in : ref_global_amax(w, rows, cols, 0);
        sg = ref_global_scale(g);
        if (global_scale_out)
            *global_scale_out = sg;
    }
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    int64_t nb = cols / block;
    for (int64_t i = 0; i < rows; i++) {
        load_row(w + i * cols, cols, 0, y);
        for (int64_t b = 0; b < nb; b++) {
            const float* yb = y + b * block;
            float amax = 0.0f;
            for (int j = 0; j < block; j++) {
                float a = fabsf(yb[j]);
                if (a > amax)
                    amax = a;
            }
            float Sdq;
            int sc;
            if (fmt == REF_FMT_MXFP4) {
                int e = ref_e8m0_exponent(amax);
                sc = e + 127;
                Sdq = (float)ldexp(1.0, e);
            } else {
                sc = nv_candidate(amax, 6.0f, sg, &Sdq);
            }
            if (scales)
                scales[i * nb + b] = (uint8_t)sc;
            for (int j = 0; j < block; j++) {
                int64_t k = i * cols + b * block + j;
                int q;
                float v;
                if (Sdq == 0.0f) {
                    q = 0;
                    v = 0.0f;
                } else {
                    float ck = ref_fp16_to_float(c[k / sub]);
                    float den = Sdq * ck;
                    float r = guarded_reciprocal(den);
                    float u = yb[j] * r;
                    q = ref_rne_e2m1(u);
                    v = (float)ref_e2m1_value(q) * Sdq;
                }
                if (w_hat_f32)
                    w_hat_f32[k] = v;
                if (w_hat_bf16)
                    w_hat_bf16[k] = ref_float_to_bf16(v);
                if (codes) {
                    if ((k & 1) == 0)
                        codes[k / 2] = (uint8_t)q;
                    else
                        codes[k / 2] = (uint8_t)(codes[k / 2] | (q << 4));
                }
            }
        }
    }
    free(y);
    return REF_OK;
}

/* FOCUS backward through the straight-through estimator (R9):
 * W_hat ~ S_dq * W / (S_dq * c_k) = W / c_k, so dL/dc_k = -sum_j g_j W_j / c_k^2,
 * summed in fp32 with the adjacent-pair tree over the sub-block.
 * [FOCUS] Metodologia §1 (STE), §3. dc: fp32 [rows, cols/sub]. */
int ref_focus_bwd(const uint16_t* w, const uint16_t* g, const uint16_t* c, int64_t rows,
                  int64_t cols, int sub, float* dc)
{
    if (rows <= 0 || cols <= 0 || sub < 1 || sub > 128 || (sub & (sub - 1)) != 0 ||
        cols % sub != 0)
        return REF_ERR_ARG;
    float p[128];
    for (int64_t k = 0; k < rows * cols / sub; k++) {
        for (int j = 0; j < sub; j++) {
            int64_t t = k * sub + j;
            p[j] = ref_bf16_to_float(g[t]) * ref_bf16_to_float(w[t]);
        }
        float acc = ref_tsum(p, sub);
        float ck = ref_fp16_to_float(c[k]);
        float cc = ck * ck;
        dc[k] = -(acc / cc);
    }
    return REF_OK;
}

/* ------------------------------------------------------------------------ */
/* FOCUS calibration: one optimizer step on the coefficients (R15, R16).     */
/* ------------------------------------------------------------------------ */

/* float -> IEEE binary16 bits, round to nearest, ties to the even bit
 * pattern; magnitudes past the largest finite half (65504) round as if 65536
 * were the next number and then become infinity. The two candidates come from
 * a binary search over the ordered positive bit patterns 0x0000..0x7BFF,
 * valued by ref_fp16_to_float. */
uint16_t ref_float_to_fp16(float v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs((double)v);
    if (isnan(v))
        return (uint16_t)(sign | 0x7E00);
    if (isinf(v))
        return (uint16_t)(sign | 0x7C00);
    int lo = 0, hi = 0x7BFF; /* largest pattern whose value is <= a */
    if (a >= (double)ref_fp16_to_float(0x7BFF)) {
        lo = 0x7BFF;
    } else {
        while (lo < hi) {
            int mid = (lo + hi + 1) / 2;
            if ((double)ref_fp16_to_float((uint16_t)mid) <= a)
                lo = mid;
            else
                hi = mid - 1;
        }
    }
    double vlo = (double)ref_fp16_to_float((uint16_t)lo);
    if (vlo == a)
        return (uint16_t)(sign | lo);
    int up = lo + 1;
    double vup = (up == 0x7C00) ? 65536.0 : (double)ref_fp16_to_float((uint16_t)up);
    double dlo = a - vlo, dup = vup - a;
    int pick;
    if (dlo < dup)
        pick = lo;
    else if (dup < dlo)
        pick = up;
    else
        pick = (lo & 1) ? up : lo;
    return (uint16_t)(sign | pick); /* pick == 0x7C00 is infinity */
}

#define REF_OPT_SGD 0
#define REF_OPT_ADAM 1

static int valid_opt(int opt, const float* m, const float* v, int64_t t)
{
    if (opt == REF_OPT_SGD)
        return 1;
    return opt == REF_OPT_ADAM && m != NULL && v != NULL && t >= 1;
}

/* Adam's step size for step t in Kingma & Ba's efficient ordering:
 * alpha_t = lr * sqrt(1 - b2^t) / (1 - b1^t), computed in double and rounded
 * once to fp32. */
static float adam_step_size(float lr, float b1, float b2, int64_t t)
{
    double bc1 = 1.0 - pow((double)b1, (double)t);
    double bc2 = 1.0 - pow((double)b2, (double)t);
    return (float)((double)lr * sqrt(bc2) / bc1);
}

/* One step on the fp32 master coefficient c of a sub-block with gradient dc
 * (R15). SGD: c <- c - lr * dc. Adam, in the efficient ordering that Kingma &
 * Ba give beside their algorithm (the bias corrections folded into the step
 * size): m <- b1 m + (1 - b1) dc; v <- b2 v + (1 - b2) dc^2;
 * c <- c - alpha_t * (m / (sqrt(v) + eps)). */
static void opt_update(int opt, float dc, float lr, float b1, float b2, float eps, float alpha,
                       float* c, float* m, float* v)
{
    if (opt == REF_OPT_SGD) {
        float step = lr * dc;
        *c = *c - step;
        return;
    }
    float om1 = 1.0f - b1;
    float om2 = 1.0f - b2;
    float m1 = b1 * (*m);
    float m2 = om1 * dc;
    float mn = m1 + m2;
    float v1 = b2 * (*v);
    float g2 = dc * dc;
    float v2 = om2 * g2;
    float vn = v1 + v2;
    float rt = sqrtf(vn);
    float den = rt + eps;
    float ratio = mn / den;
    float step = alpha * ratio;
    *m = mn;
    *v = vn;
    *c = *c - step;
}

/* The forward pass consumes the FP16 coefficient (the pages' parameter type):
 * the value of the master coefficient rounded to half precision. */
static float coefficient_used(float c32)
{
    return ref_fp16_to_float(ref_float_to_fp16(c32));
}

/* FOCUS coefficient update from an external gradient g = dL/dW_hat (for a
 * loss the caller differentiates: the pages' distillation loss, or a layer
 * output loss): the straight-through gradient of R9 at the coefficient the
 * forward used, then one optimizer step on the master coefficients.
 * c (fp32 master), m, v: [rows, cols/sub], updated in place; c_half: fp16
 * bits of the updated coefficients, nullable. [FOCUS] Metodologia §1 (STE
 * and gradient descent on the scales), §2 (c as FP16 learnable parameter). */
int ref_focus_update(const uint16_t* w, const uint16_t* g, float* c, uint16_t* c_half,
                     float* m, float* v, int64_t rows, int64_t cols, int sub, int opt, float lr,
                     float b1, float b2, float eps, int64_t t)
{
    if (rows <= 0 || cols <= 0 || sub < 1 || sub > 128 || (sub & (sub - 1)) != 0 ||
        cols % sub != 0 || !valid_opt(opt, m, v, t))
        return REF_ERR_ARG;
    float alpha = opt == REF_OPT_ADAM ? adam_step_size(lr, b1, b2, t) : lr;
    float p[128];
    for (int64_t k = 0; k < rows * cols / sub; k++) {
        for (int j = 0; j < sub; j++) {
            int64_t e = k * sub + j;
            p[j] = ref_bf16_to_float(g[e]) * ref_bf16_to_float(w[e]);
        }
        float acc = ref_tsum(p, sub);
        float ck = coefficient_used(c[k]);
        float cc = ck * ck;
        float dc = -(acc / cc);
        opt_update(opt, dc, lr, b1, b2, eps, alpha, &c[k], m ? &m[k] : NULL,
                   v ? &v[k] : NULL);
        if (c_half)
            c_half[k] = ref_float_to_fp16(c[k]);
    }
    return REF_OK;
}

/* One calibration step on the weight-reconstruction loss L = sum (W_hat - W)^2
 * (R16): the FOCUS forward at the coefficients used, the loss gradient
 * g = 2 (W_hat - W) in fp32 (W_hat not rounded to bf16), the straight-through
 * coefficient gradient dc = -(tsum(g * W) / c^2), one optimizer step.
 * sse (nullable, fp32 [rows, cols/sub]) receives tsum((W_hat - W)^2) per
 * sub-block, before the step. [FOCUS] Metodologia §1-§3. */
int ref_focus_step(const uint16_t* w, int64_t rows, int64_t cols, int fmt, int block, int sub,
                   const float* global_amax_in, float* global_scale_out, float* c,
                   uint16_t* c_half, float* m, float* v, float* sse, int opt, float lr, float b1,
                   float b2, float eps, int64_t t)
{
    if (!valid_common(rows, cols, fmt, block, 0))
        return REF_ERR_ARG;
    if (fmt == REF_FMT_UE5M3)
        return REF_ERR_ARG; /* FOCUS is defined for MXFP4 and NVFP4 */
    if (sub < 1 || block % sub != 0 || (sub & (sub - 1)) != 0 || !valid_opt(opt, m, v, t))
        return REF_ERR_ARG;
    float sg = 1.0f;
    if (fmt == REF_FMT_NVFP4) {
        float ga = global_amax_in ? *global_amax_in : ref_global_amax(w, rows, cols, 0);
        sg = ref_global_scale(ga);
        if (global_scale_out)
            *global_scale_out = sg;
    }
    float alpha = opt == REF_OPT_ADAM ? adam_step_size(lr, b1, b2, t) : lr;
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    float d[128], p[128];
    int64_t nb = cols / block;
    for (int64_t i = 0; i < rows; i++) {
        load_row(w + i * cols, cols, 0, y);
        for (int64_t b = 0; b < nb; b++) {
            const float* yb = y + b * block;
            float amax = 0.0f;
            for (int j = 0; j < block; j++) {
                float a = fabsf(yb[j]);
                if (a > amax)
                    amax = a;
            }
            float Sdq;
            if (fmt == REF_FMT_MXFP4)
                Sdq = (float)ldexp(1.0, ref_e8m0_exponent(amax));
            else
                (void)nv_candidate(amax, 6.0f, sg, &Sdq);
            for (int s0 = 0; s0 < block; s0 += sub) {
                int64_t k = (i * cols + b * block + s0) / sub;
                float ck = coefficient_used(c[k]);
                for (int j = 0; j < sub; j++) {
                    float wj = yb[s0 + j];
                    float what = 0.0f;
                    if (Sdq != 0.0f) {
                        float den = Sdq * ck;
                        float r = guarded_reciprocal(den);
                        float u = wj * r;
                        what = (float)ref_e2m1_value(ref_rne_e2m1(u)) * Sdq;
                    }
                    d[j] = what - wj;
                    float gj = d[j] + d[j];
                    p[j] = gj * wj;
                }
                if (sse) {
                    float e[128];
                    for (int j = 0; j < sub; j++)
                        e[j] = d[j] * d[j];
                    sse[k] = ref_tsum(e, sub);
                }
                float acc = ref_tsum(p, sub);
                float cc = ck * ck;
                float dc = -(acc / cc);
                opt_update(opt, dc, lr, b1, b2, eps, alpha, &c[k], m ? &m[k] : NULL,
                           v ? &v[k] : NULL);
                if (c_half)
                    c_half[k] = ref_float_to_fp16(c[k]);
            }
        }
    }
    free(y);
    return REF_OK;
}

/* ------------------------------------------------------------------------ */
/* Element-wise array forms of the rounding functions, for exhaustive checks. */
/* ------------------------------------------------------------------------ */

void ref_rne_e2m1_array(const float* u, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)ref_rne_e2m1(u[i]);
}

void ref_rne_e4m3_array(const float* v, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)ref_rne_e4m3_sat(v[i]);
}

/* Rounds the fp32 numbers whose bit patterns are first, first+1, ...,
 * first+n-1 (no input array needed for sweeps over bit patterns). */
void ref_rne_e2m1_bits_range(uint32_t first, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)ref_rne_e2m1(bits2f(first + (uint32_t)i));
}

void ref_rne_e4m3_bits_range(uint32_t first, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)ref_rne_e4m3_sat(bits2f(first + (uint32_t)i));
}

void ref_rne_ue5m3_array(const float* v, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)ref_rne_ue5m3_sat(v[i]);
}

void ref_rne_ue5m3_bits_range(uint32_t first, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = (uint8_t)ref_rne_ue5m3_sat(bits2f(first + (uint32_t)i));
}

void ref_fwht_array(float* t, int64_t n_chunks, int n)
{
    for (int64_t i = 0; i < n_chunks; i++)
        ref_fwht(t + i * n, n);
}
