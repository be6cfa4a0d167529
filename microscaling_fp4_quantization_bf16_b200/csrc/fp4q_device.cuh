// fp4q_device.cuh -- device primitives shared by the sm_100a kernels.
//
// Every floating-point step is an explicit round-to-nearest-even IEEE
// binary32 operation (__fadd_rn, __fmul_rn, __fdiv_rn, __frcp_rn: never
// contracted into FMA) or a hardware conversion instruction (cvt with .rn and
// .satfinite), so a kernel's result is a fixed function of its input:
//  - E2M1 encode: cvt.rn.satfinite.e2m1x2.f32 (RNE, ties to the even
//    mantissa, saturating at +-6, sign kept);
//  - E2M1 decode: cvt.rn.f16x2.e2m1x2 then f16 -> f32 (both exact);
//  - E4M3 encode: cvt.rn.satfinite.e4m3x2.f32 (RNE, saturating at 448);
//  - E4M3 decode: cvt.rn.f16x2.e4m3x2 then f16 -> f32 (exact).
// Formats: OCP E2M1 / E4M3 ("Finer is Better (with the Right Scaling)",
// 手法 1 and 意義と主張), E8M0 ("Bridging the Gap Between Promise and
// Performance for Microscaling FP4 Quantization", 技術概要 §1).
#pragma once

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace fp4q {

// Elements owned by one thread: 32 contiguous elements of the flattened
// tensor (64 bytes of bf16 = four 128-bit loads). Blocks (4..32) and Hadamard
// chunks (16, 32) lie inside a segment; 64/128-wide chunks span 2/4 lanes.
constexpr int SEG = 32;

// Calls f(std::integral_constant<int, i>{}) for i = 0 .. N-1, so that i is a
// compile-time constant inside f (register arrays stay in registers).
template <int N, int I = 0, class F>
__device__ __forceinline__ void static_for(F&& f)
{
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        static_for<N, I + 1>(f);
    }
}

// ------------------------------------------------------------------ launch

// Programmatic dependent launch. Every kernel of the library is launched with
// programmatic stream serialization and starts with pdl_begin(): it waits
// until the previous kernel in the stream has completed and its writes are
// visible (so reading inputs it produced is safe), then lets the next kernel
// begin launching, which overlaps that launch with this kernel's execution.
__device__ __forceinline__ void pdl_begin()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ loads

__device__ __forceinline__ uint4 ldg_stream(const uint4* p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

#ifndef FP4Q_UNPACK_PRMT
#define FP4Q_UNPACK_PRMT 1
#endif
// The low bf16 of a word, widened: the byte permute keeps it on the integer
// ALU (a shift may be issued to the FMA pipe as a multiply).
__device__ __forceinline__ float bf_lo(uint32_t w)
{
#if FP4Q_UNPACK_PRMT
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, 0x1044;" : "=r"(r) : "r"(w));
    return __uint_as_float(r);
#else
    return __uint_as_float(w << 16);
#endif
}
// The high bf16 of a word, widened: a mask on the integer ALU, or (MIXED)
// the mixed-precision add of -0, which widens the bf16 operand exactly and
// runs on the floating-point pipes. The NVFP4 / UE5M3 quantize kernels take
// the add (measured: 4-over-6 on the 16384 x 8192 activations 104.6 -> 102.6
// us, bit-identical output); MXFP4 keeps the mask (the add measured 1% slower
// there).
template <bool MIXED = false>
__device__ __forceinline__ float bf_hi(uint32_t w)
{
    if constexpr (MIXED) {
        float r;
        asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %1;\n\tadd.rn.f32.bf16 %0, b, %2;\n\t}"
            : "=f"(r)
            : "r"(w), "f"(-0.0f));
        return r;
    } else {
        return __uint_as_float(w & 0xFFFF0000u);
    }
}

// Raw bf16 words of segment s (elements s*32 .. s*32+31) of an array of n
// elements: element 2i in the low half of word i. Elements at or beyond n
// read as +0. Issuing these loads early lets a kernel overlap their latency
// with other start-up work before unpacking.
__device__ __forceinline__ void load_seg_raw(const uint16_t* x, int64_t n, int64_t s, uint4 (&v)[4])
{
    const int64_t base = s * SEG;
    if (base + SEG <= n) {
        const uint4* p = reinterpret_cast<const uint4*>(x + base);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[k] = ldg_stream(p + k);
    } else {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t lo = (base + 2 * i < n) ? (uint32_t)x[base + 2 * i] : 0u;
            const uint32_t hi = (base + 2 * i + 1 < n) ? (uint32_t)x[base + 2 * i + 1] : 0u;
            w[i] = lo | (hi << 16);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    }
}

// bf16 words -> fp32 values (exact).
template <bool MIXED_HI = false>
__device__ __forceinline__ void unpack_seg(const uint4 (&v)[4], float (&y)[SEG])
{
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        y[8 * k + 0] = bf_lo(v[k].x);
        y[8 * k + 1] = bf_hi<MIXED_HI>(v[k].x);
        y[8 * k + 2] = bf_lo(v[k].y);
        y[8 * k + 3] = bf_hi<MIXED_HI>(v[k].y);
        y[8 * k + 4] = bf_lo(v[k].z);
        y[8 * k + 5] = bf_hi<MIXED_HI>(v[k].z);
        y[8 * k + 6] = bf_lo(v[k].w);
        y[8 * k + 7] = bf_hi<MIXED_HI>(v[k].w);
    }
}

// Loads segment s of a bf16 array of n elements, widened to fp32 (exact).
// Elements at or beyond n read as +0.
__device__ __forceinline__ void load_seg_bf16(const uint16_t* x, int64_t n, int64_t s, float (&y)[SEG])
{
    uint4 v[4];
    load_seg_raw(x, n, s, v);
    unpack_seg(v, y);
}

// ------------------------------------------------------------------ E2M1

// u[0..7] -> eight 4-bit codes; element j in bits 4j..4j+3. In
// cvt.rn.satfinite.e2m1x2.f32 d, a, b the first source a lands in the upper
// nibble, so element 2j+1 is passed first.
__device__ __forceinline__ uint32_t e2m1_pack8(const float* u)
{
    uint32_t r;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(r)
        : "f"(u[0]), "f"(u[1]), "f"(u[2]), "f"(u[3]), "f"(u[4]), "f"(u[5]), "f"(u[6]), "f"(u[7]));
    return r;
}

// u[0..3] -> four 4-bit codes in bits 0..15 (element j in bits 4j..4j+3).
__device__ __forceinline__ uint32_t e2m1_pack4(const float* u)
{
    uint32_t r;
    asm("{\n\t.reg .b8 q0, q1;\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "mov.b16 t, {q0, q1};\n\t"
        "cvt.u32.u16 %0, t;\n\t}"
        : "=r"(r)
        : "f"(u[0]), "f"(u[1]), "f"(u[2]), "f"(u[3]));
    return r;
}

// f16 pair -> two floats, exactly: v + (-0) in the mixed-precision add, whose
// f16 operand is widened exactly; adding -0 changes no value (+0 + -0 = +0
// under round-to-nearest). Measured 2% faster than the plain conversion in
// the quantize kernels, whose FMA-heavy pipe the plain conversion loads.
__device__ __forceinline__ float2 h2_to_f2(uint32_t h)
{
    float lo, hi;
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "add.rn.f32.f16 %0, a, %3;\n\t"
        "add.rn.f32.f16 %1, b, %3;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h), "f"(-0.0f));
    return make_float2(lo, hi);
}

// Eight 4-bit codes (element j in bits 4j..4j+3) -> their exact values.
__device__ __forceinline__ void e2m1_unpack8(uint32_t q, float* v)
{
    uint32_t h0, h1, h2, h3;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "mov.b32 {q0, q1, q2, q3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, q2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, q3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(q));
    float2 f;
    f = h2_to_f2(h0); v[0] = f.x; v[1] = f.y;
    f = h2_to_f2(h1); v[2] = f.x; v[3] = f.y;
    f = h2_to_f2(h2); v[4] = f.x; v[5] = f.y;
    f = h2_to_f2(h3); v[6] = f.x; v[7] = f.y;
}

// Four 4-bit codes in bits 0..15 -> their exact values.
__device__ __forceinline__ void e2m1_unpack4(uint32_t q, float* v)
{
    uint32_t h0, h1;
    unsigned short t = (unsigned short)(q & 0xFFFFu);
    asm("{\n\t.reg .b8 q0, q1;\n\t"
        "mov.b16 {q0, q1}, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t}"
        : "=r"(h0), "=r"(h1)
        : "h"(t));
    float2 f;
    f = h2_to_f2(h0); v[0] = f.x; v[1] = f.y;
    f = h2_to_f2(h1); v[2] = f.x; v[3] = f.y;
}

// ------------------------------------------------------------------ E4M3

// Two non-negative floats -> two E4M3 bytes: lo in bits 0-7, hi in bits 8-15.
__device__ __forceinline__ uint32_t e4m3_enc2(float hi, float lo)
{
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t e4m3_enc(float v) { return e4m3_enc2(0.0f, v) & 0xFFu; }

// E4M3 byte (0..0x7E) -> exact value.
__device__ __forceinline__ float e4m3_dec(uint32_t code)
{
    uint32_t h;
    unsigned short c = (unsigned short)(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
    return h2_to_f2(h).x;
}

// ------------------------------------------------------------------ UE5M3

// UE5M3 scale byte -> exact value: unsigned, 5 exponent bits with bias 15,
// 3 mantissa bits, exponent field 0 subnormal (m * 2^-17); 0xFF is NaN.
__device__ __forceinline__ float ue5m3_dec(uint32_t c)
{
    if (c >= 0xFFu)
        return __uint_as_float(0x7FC00000u);
    if (c < 8u)
        return __fmul_rn((float)c, 0x1p-17f);  // exact
    return __uint_as_float((((c >> 3) + 112u) << 23) | ((c & 7u) << 20));
}

// v >= 0 -> the nearest UE5M3 byte, ties to the even code, saturating at
// 0xFE. Below 2^-14 the step is 2^-17: v * 2^17 is exact and rounded to the
// nearest even integer (8 is the first normal code). Above, the fp32
// significand is rounded to 3 bits at bit 20 (ties to even, the carry moving
// into the exponent), then re-biased from 127 to 15.
__device__ __forceinline__ uint32_t ue5m3_enc(float v)
{
    const uint32_t b = __float_as_uint(v);
    if (b < 0x38800000u)  // v < 2^-14
        return (uint32_t)__float2int_rn(__fmul_rn(v, 0x1p17f));
    const uint32_t r = (b + 0x7FFFFu + ((b >> 20) & 1u)) >> 20;
    return min(r - (112u << 3), 0xFEu);
}

// ------------------------------------------------------------------ scales

// FP32 global scale of hierarchical scaling: amax / (448 * 6); 1 when that is
// not a positive finite number.
__device__ __forceinline__ float global_scale_of(float g)
{
    float sg = __fdiv_rn(g, 2688.0f);
    if (!(sg > 0.0f) || !(g <= FLT_MAX))
        sg = 1.0f;
    return sg;
}

// 1 / S, with an overflowing reciprocal replaced by the largest finite float
// of the same sign.
__device__ __forceinline__ float guarded_rcp(float S)
{
    float r = __frcp_rn(S);
    if (fabsf(r) > FLT_MAX)
        r = copysignf(FLT_MAX, r);
    return r;
}

// E8M0 exponent of a block abs-max a >= 0: floor(log2 a) - 2 clamped to
// [-127, 127] (a == 0 -> -127). For a biased fp32 exponent E (0 for zero and
// subnormals) this is max(E - 129, -127): subnormal a has floor(log2 a) <= -127.
__device__ __forceinline__ int e8m0_exp(float a)
{
    int E = (int)((__float_as_uint(a) >> 23) & 0xFFu);
    return max(E - 129, -127);
}

// E8M0 byte -> 2^(b - 127); 255 is NaN; byte 0 is the subnormal 2^-127.
__device__ __forceinline__ float e8m0_dec(uint32_t b)
{
    if (b == 255u)
        return __uint_as_float(0x7FC00000u);
    return b == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(b << 23);
}

// Per-thread constants of E4M3 scale selection for target T in {6, 4}:
// den_T = T * s_g and its correctly rounded reciprocal.
struct NvConsts {
    float den6, rden6, den4, rden4;
    bool fast;  // both reciprocals finite: the quotient shortcut applies
    // 2^-105 <= s_g <= 2^110: every nonzero scale S = E4M3(c) s_g lies in
    // (2^-120, 2^119], so a power-of-two rotation factor k >= 2^-3 can be
    // folded into fl(1/S) exactly (see candidate_seg and fold_ok below).
    bool fold;
};

__device__ __forceinline__ NvConsts nv_consts(float sg)
{
    NvConsts k;
    k.den6 = __fmul_rn(6.0f, sg);
    k.den4 = __fmul_rn(4.0f, sg);
    k.rden6 = __frcp_rn(k.den6);
    k.rden4 = __frcp_rn(k.den4);
    k.fast = k.rden6 <= FLT_MAX && k.rden4 <= FLT_MAX;
    k.fold = sg >= 0x1p-105f && sg <= 0x1p110f;
    return k;
}

// 2^e for e in [-127, 127] (2^-127 is the subnormal 0x00400000 = 2^22 * 2^-149).
__device__ __forceinline__ float pow2f(int e)
{
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// ------------------------------------------------------------------ Hadamard

template <int N>
struct HadK;
template <> struct HadK<16> { static constexpr float k = 0x1p-2f; };
template <> struct HadK<32> { static constexpr float k = 0x1.6a09e6p-3f; };
template <> struct HadK<64> { static constexpr float k = 0x1p-3f; };
template <> struct HadK<128> { static constexpr float k = 0x1.6a09e6p-4f; };

// Packed pairs of fp32 (sm_100 add/sub/mul.rn.f32x2: two IEEE round-to-
// nearest-even operations, no flush-to-zero, one instruction).
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pk2(float lo, float hi)
{
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void upk2(f32x2 v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Scale codes c[i] = RNE_E4M3_sat(fl(a[i] / den[i])), a[i] >= 0, mostly
// without a division. q = fl(a * fl(1/den)) is within a few units in the last
// place of fl(a / den) (two roundings of relative size <= 2^-24 each), so the
// two round to different E4M3 codes only if an E4M3 rounding boundary (a
// midpoint between adjacent E4M3 values) lies within that distance of q. The
// check rounds q * (1 - 2^-18) and q * (1 + 2^-18), which bracket both q and
// fl(a / den) by a wide margin: if their codes agree, no midpoint lies between
// them and code(q) is the code of fl(a / den) (E4M3 rounding is monotone). If
// they disagree, that pair's codes are recomputed from the IEEE division. q = 0
// and q = inf (saturating like any q > 448) need no special case. Quotients
// are formed and checked two at a time (packed multiplies, one conversion of
// two values).
template <int N>
__device__ __forceinline__ void e4m3_quotient_codes(const float (&a)[N], const float (&den)[N],
                                                    const float (&rden)[N], bool fast,
                                                    uint32_t (&c)[N])
{
    constexpr int NP = (N + 1) / 2;
    const f32x2 up = pk2(1.0f + 0x1p-18f, 1.0f + 0x1p-18f);
    const f32x2 dn = pk2(1.0f - 0x1p-18f, 1.0f - 0x1p-18f);
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int i = 2 * p, j = 2 * p + 1 < N ? 2 * p + 1 : 2 * p;
        const f32x2 Q = mul2(pk2(a[i], a[j]), pk2(rden[i], rden[j]));
        float q0, q1, p0, p1, m0, m1;
        upk2(Q, q0, q1);
        upk2(mul2(Q, up), p0, p1);
        upk2(mul2(Q, dn), m0, m1);
        uint32_t cq = e4m3_enc2(q1, q0);
        // a midpoint between the brackets (or no fast path at all): this pair
        // takes the IEEE division. Quotients that share a segment rarely need
        // it together, so each pair branches on its own.
        if (!fast || e4m3_enc2(p1, p0) != e4m3_enc2(m1, m0))
            cq = e4m3_enc2(__fdiv_rn(a[j], den[j]), __fdiv_rn(a[i], den[i]));
        c[i] = cq & 0xFFu;
        if (2 * p + 1 < N)
            c[j] = cq >> 8;
    }
}

__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c)
{
    f32x2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Normalised Walsh-Hadamard transform of every ROT-wide chunk of a segment:
// stages h = 1, 2, 4, ... in ascending order, (t[i], t[i+h]) <- (t[i]+t[i+h],
// t[i]-t[i+h]), then one multiply by k_ROT. All stages run on packed pairs
// P[i] = {y[i], y[i + 16]}:
//  - h < 16: both lanes of one add.f32x2 / sub.f32x2 are butterflies of the
//    same stage;
//  - h = 16 pairs the two lanes of P[i]: fma(P, {1, -1}, {y[i+16], y[i]})
//    gives {y[i] + y[i+16], y[i] - y[i+16]}, each product exact and the sum
//    rounded once, so bit for bit the add and the subtract;
//  - h = 32, 64 pair lane L with lane L ^ (h / 32): the lower lane needs
//    p + v, the upper p - v (p the partner's value, v its own), again one
//    exact product and one rounding: fma(+-1, v, p).
// All 32 lanes of the warp must call this together. SCALE = false leaves
// out the multiply by k_ROT (the caller applies it, or folds it where k_ROT is
// a power of two: see candidate_seg).
template <int ROT, bool SCALE = true>
__device__ __forceinline__ void rotate_seg(float (&y)[SEG], int lane)
{
    if constexpr (ROT > 0) {
        constexpr int LOCAL = ROT < SEG ? ROT : SEG;
        f32x2 P[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            P[i] = pk2(y[i], y[i + 16]);
#pragma unroll
        for (int h = 1; h < (LOCAL < 16 ? LOCAL : 16); h <<= 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if ((i & h) == 0) {
                    f32x2 a = P[i], b = P[i + h];
                    P[i] = add2(a, b);
                    P[i + h] = sub2(a, b);
                }
            }
        }
        if constexpr (LOCAL == SEG) {  // stage 16
            const f32x2 pm = pk2(1.0f, -1.0f);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float lo, hi;
                upk2(P[i], lo, hi);
                P[i] = fma2(P[i], pm, pk2(hi, lo));
            }
        }
#pragma unroll
        for (int h = SEG; h < ROT; h <<= 1) {
            const int lm = h / SEG;
            const float sgn = (lane & lm) == 0 ? 1.0f : -1.0f;
            const f32x2 ss = pk2(sgn, sgn);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float lo, hi;
                upk2(P[i], lo, hi);
                const float plo = __shfl_xor_sync(0xFFFFFFFFu, lo, lm);
                const float phi = __shfl_xor_sync(0xFFFFFFFFu, hi, lm);
                P[i] = fma2(ss, P[i], pk2(plo, phi));
            }
        }
        if constexpr (SCALE) {
            const f32x2 kk = pk2(HadK<ROT>::k, HadK<ROT>::k);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                upk2(mul2(P[i], kk), y[i], y[i + 16]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                upk2(P[i], y[i], y[i + 16]);
        }
    }
}

// y <- y * k_ROT for a segment left unscaled by rotate_seg<ROT, false>.
template <int ROT>
__device__ __forceinline__ void scale_seg(float (&y)[SEG])
{
    const f32x2 kk = pk2(HadK<ROT>::k, HadK<ROT>::k);
#pragma unroll
    for (int i = 0; i < 16; ++i)
        upk2(mul2(pk2(y[i], y[i + 16]), kk), y[i], y[i + 16]);
}

// Segments per thread (one; kept as a parameter of the kernels' indexing).
// Two segments per thread for 64/128-wide rotations (all stages up to 32 in
// registers) measured slower on B200 than one segment with shuffle stages.
template <int ROT>
struct SegsPerThread {
    static constexpr int value = 1;
};

// Loads the segment(s) of thread t and rotates them.
template <int ROT>
__device__ __forceinline__ void load_rotate(const uint16_t* x, int64_t n, int64_t t, int lane,
                                            float (&y)[SegsPerThread<ROT>::value][SEG])
{
    load_seg_bf16(x, n, t, y[0]);
    rotate_seg<ROT>(y[0], lane);
}

// ------------------------------------------------------------------ blocks

// Abs-max of each B-wide block of the segment (exact: max is order-free).
template <int B>
__device__ __forceinline__ void block_amax(const float (&y)[SEG], float (&a)[SEG / B])
{
#pragma unroll
    for (int b = 0; b < SEG / B; ++b) {
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < B; ++j)
            m = fmaxf(m, fabsf(y[b * B + j]));
        a[b] = m;
    }
}

// Adjacent-pair tree sum of e[off .. off+B): for h = 1, 2, .., B/2,
// e[i] += e[i + h] for i = off, off + 2h, ...
template <int B>
__device__ __forceinline__ float tree_sum(float* e)
{
#pragma unroll
    for (int h = 1; h < B; h <<= 1) {
#pragma unroll
        for (int i = 0; i + h < B; i += 2 * h)
            e[i] = __fadd_rn(e[i], e[i + h]);
    }
    return e[0];
}

// Codes of the segment: u = y * r(block), RNE to E2M1, eight per word; the
// codes of blocks with a zero scale are forced to 0x0.
//
// `keep` must be a run-time all-ones word (a kernel argument). Every encoded
// word is ANDed with it before anything decodes it again: decoding a word
// straight out of e2m1_pack8, with no intervening run-time operation, was
// measured on sm_100a to return 0 for the elements held in bytes 2 and 3.
template <int B>
__device__ __forceinline__ void encode_seg_packed(const float (&y)[SEG], const float (&r)[SEG / B],
                                           const bool (&zero)[SEG / B], uint32_t keep,
                                           uint32_t (&q)[4])
{
    // u = y * r on packed pairs {i, i + 16}: words w and w + 2 together
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        float u[8], v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = 8 * w + j;
            f32x2 U = mul2(pk2(y[i], y[i + 16]), pk2(r[i / B], r[(i + 16) / B]));
            upk2(U, u[j], v[j]);
        }
        uint32_t m0 = 0, m1 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (zero[(8 * w + j) / B])
                m0 |= 0xFu << (4 * j);
            if (zero[(8 * w + 16 + j) / B])
                m1 |= 0xFu << (4 * j);
        }
        q[w] = e2m1_pack8(u) & (keep & ~m0);
        q[w + 2] = e2m1_pack8(v) & (keep & ~m1);
    }
}

// Dequantized values of the segment: value(code) * S(block).
template <int B>
__device__ __forceinline__ void decode_seg(const uint32_t (&q)[4], const float (&S)[SEG / B],
                                           float (&yh)[SEG])
{
    float v[SEG];
#pragma unroll
    for (int w = 0; w < 4; ++w)
        e2m1_unpack8(q[w], v + 8 * w);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        f32x2 Y = mul2(pk2(v[i], v[i + 16]), pk2(S[i / B], S[(i + 16) / B]));
        upk2(Y, yh[i], yh[i + 16]);
    }
}

// Per-block SSE of y against value(code) * S, tree-summed. Values are formed
// on packed pairs {i, i + 16}: for B <= 16 the two lanes of E[g*B .. g*B + B)
// hold two whole blocks (g and g + 16/B) whose adjacent-pair trees run in
// lockstep; for B = 32 the packed tree yields the two half sums and the last
// level adds them, which is the same tree.
//
// ptxas fuses a packed multiply (mul.rn.f32x2, and even fma.rn.f32x2 with a
// -0 addend) into a following packed add/sub although .rn and -fmad=false
// forbid contraction; measured on sm_100a it changed low bits. A packed
// product is therefore always consumed first by a scalar __fsub_rn /
// __fadd_rn, which are never contracted: d = y - yhat and the first tree level.
template <int B>
__device__ __forceinline__ void sse_seg_packed(const float (&y)[SEG], const uint32_t (&q)[4],
                                        const float (&S)[SEG / B], float (&sse)[SEG / B])
{
    float v[SEG];
#pragma unroll
    for (int w = 0; w < 4; ++w)
        e2m1_unpack8(q[w], v + 8 * w);
    float e[SEG];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float h0, h1, d0, d1;
        upk2(mul2(pk2(v[i], v[i + 16]), pk2(S[i / B], S[(i + 16) / B])), h0, h1);
        d0 = __fsub_rn(y[i], h0);
        d1 = __fsub_rn(y[i + 16], h1);
        upk2(mul2(pk2(d0, d1), pk2(d0, d1)), e[i], e[i + 16]);
    }
    f32x2 E[8];  // tree level h = 1, scalar: E[j] = {e[2j] + e[2j+1], e[2j+16] + e[2j+17]}
#pragma unroll
    for (int j = 0; j < 8; ++j)
        E[j] = pk2(__fadd_rn(e[2 * j], e[2 * j + 1]), __fadd_rn(e[2 * j + 16], e[2 * j + 17]));
    constexpr int G = B < 16 ? B : 16;  // packed tree width (elements)
#pragma unroll
    for (int h = 1; h < G / 2; h <<= 1) {  // levels 2 .. G/2 on the half-length array
#pragma unroll
        for (int j = 0; j + h < 8; j += 2 * h)
            E[j] = add2(E[j], E[j + h]);
    }
    if constexpr (B == 32) {
        float lo, hi;
        upk2(E[0], lo, hi);
        sse[0] = __fadd_rn(lo, hi);
    } else {
#pragma unroll
        for (int g = 0; g < 16 / B; ++g)
            upk2(E[g * B / 2], sse[g], sse[g + 16 / B]);
    }
}

// Scalar forms of encode_seg and sse_seg (one IEEE operation per element
// and step); the packed forms above compute the same bits.
template <int B>
__device__ __forceinline__ void encode_seg_scalar(const float (&y)[SEG], const float (&r)[SEG / B],
                                                  const bool (&zero)[SEG / B], uint32_t keep,
                                                  uint32_t (&q)[4])
{
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        float u[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            u[j] = __fmul_rn(y[8 * w + j], r[(8 * w + j) / B]);
        uint32_t qw = e2m1_pack8(u);
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (zero[(8 * w + j) / B])
                m |= 0xFu << (4 * j);
        q[w] = qw & (keep & ~m);
    }
}

template <int B>
__device__ __forceinline__ void sse_seg_scalar(const float (&y)[SEG], const uint32_t (&q)[4],
                                               const float (&S)[SEG / B], float (&sse)[SEG / B])
{
    float e[SEG];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        float v[8];
        e2m1_unpack8(q[w], v);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = 8 * w + j;
            float d = __fsub_rn(y[i], __fmul_rn(v[j], S[i / B]));
            e[i] = __fmul_rn(d, d);
        }
    }
#pragma unroll
    for (int b = 0; b < SEG / B; ++b)
        sse[b] = tree_sum<B>(e + b * B);
}

// Word-pair forms for blocks of B <= 8 elements: words w and w + 2 of a
// segment (elements 8w .. 8w+7 and 8w+16 .. 8w+23) hold 8 / B whole blocks
// each, so a segment can be processed in two halves. Element j of the half is
// packed with element j of the other word (the pairs {i, i + 16} of the
// segment forms above), and every result equals the segment forms' bits.
template <int B>
__device__ __forceinline__ void encode_word_pair(const float (&y)[SEG], int w, const float (&rl)[8 / B],
                                                 const float (&rh)[8 / B], uint32_t zl, uint32_t zh,
                                                 uint32_t keep, uint32_t& ql, uint32_t& qh)
{
    float u[8], v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = 8 * w + j;
        upk2(mul2(pk2(y[i], y[i + 16]), pk2(rl[j / B], rh[j / B])), u[j], v[j]);
    }
    ql = e2m1_pack8(u) & (keep & ~zl);
    qh = e2m1_pack8(v) & (keep & ~zh);
}

template <int B>
__device__ __forceinline__ void sse_word_pair(const float (&y)[SEG], int w, uint32_t ql, uint32_t qh,
                                              const float (&Sl)[8 / B], const float (&Sh)[8 / B],
                                              float (&el)[8 / B], float (&eh)[8 / B])
{
    static_assert(B == 4 || B == 8, "word pairs hold whole blocks of 4 or 8");
    float va[8], vb[8], e[16];
    e2m1_unpack8(ql, va);
    e2m1_unpack8(qh, vb);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = 8 * w + j;
        float h0, h1;
        upk2(mul2(pk2(va[j], vb[j]), pk2(Sl[j / B], Sh[j / B])), h0, h1);
        const float d0 = __fsub_rn(y[i], h0);
        const float d1 = __fsub_rn(y[i + 16], h1);
        upk2(mul2(pk2(d0, d1), pk2(d0, d1)), e[j], e[8 + j]);
    }
    f32x2 E[4];  // first tree level, scalar: {e[2k] + e[2k+1] of word w, same of word w + 2}
#pragma unroll
    for (int k = 0; k < 4; ++k)
        E[k] = pk2(__fadd_rn(e[2 * k], e[2 * k + 1]), __fadd_rn(e[8 + 2 * k], e[8 + 2 * k + 1]));
    E[0] = add2(E[0], E[1]);
    E[2] = add2(E[2], E[3]);
    if constexpr (B == 4) {
        upk2(E[0], el[0], eh[0]);
        upk2(E[2], el[1], eh[1]);
    } else {
        upk2(add2(E[0], E[2]), el[0], eh[0]);
    }
}

// Selected forms (both compute the same bits). The packed encode measured
// faster in the MXFP4 kernel and slower in the NVFP4 ones (register
// pressure), so the quantize kernel picks it per format.
#ifndef FP4Q_PACKED_ENCODE
#define FP4Q_PACKED_ENCODE 0
#endif
#ifndef FP4Q_PACKED_SSE
#define FP4Q_PACKED_SSE 1
#endif

template <int B, bool PACKED = FP4Q_PACKED_ENCODE>
__device__ __forceinline__ void encode_seg(const float (&y)[SEG], const float (&r)[SEG / B],
                                           const bool (&zero)[SEG / B], uint32_t keep,
                                           uint32_t (&q)[4])
{
    if constexpr (PACKED)
        encode_seg_packed<B>(y, r, zero, keep, q);
    else
        encode_seg_scalar<B>(y, r, zero, keep, q);
}

template <int B>
__device__ __forceinline__ void sse_seg(const float (&y)[SEG], const uint32_t (&q)[4],
                                        const float (&S)[SEG / B], float (&sse)[SEG / B])
{
    if constexpr (FP4Q_PACKED_SSE)
        sse_seg_packed<B>(y, q, S, sse);
    else
        sse_seg_scalar<B>(y, q, S, sse);
}

// One candidate scale per block for a whole segment: the packed E2M1 codes
// (before zero-scale masking) and, with WANT_SSE, each block's SSE -- the
// adjacent-pair tree sum of fl(d^2), d = fl(y - fl(value(q) * S)).
//
// t holds y (FOLD = false), or the rotated values before their multiply by
// k = kf, a power of two (FOLD = true): then y = t * kf exactly, r must
// already be fl(1/S) * kf (exact), u = fl(t * r) = fl(y * fl(1/S)) and
// d = fma(t, kf, -yhat) = fl(y - yhat); the caller guarantees the exactness
// conditions (no value of t * kf or fl(1/S) * kf is lost to underflow where it
// matters).
//
// Words w and w + 2 are processed together on packed pairs {i, i + 16}. The
// products that feed a subtraction or a tree addition are formed as
// fma(a, b, z) with z a run-time +0 (kernel argument): fl(a * b + 0) equals
// fl(a * b) (a zero product gives +0, which changes no difference or square
// below), and ptxas cannot contract such an fma into the following packed
// add, which it does with a packed multiply. nS holds -S per block, so
// fma(v, -S, z) = -yhat and d = y + (-yhat).
#ifndef FP4Q_CAND_SCALAR
#define FP4Q_CAND_SCALAR 0
#endif

template <int B>
__host__ __device__ constexpr int blocks_per_word() { return B < 8 ? 8 / B : 1; }

// Words w and w + 2 of candidate_seg: rl / rh and nSl / nSh hold r and -S of
// the blocks that word w and word w + 2 touch (8 / B blocks each for B <= 8,
// else the one block each). Returns their codes qa, qb and, with WANT_SSE,
// the block SSEs el / eh for B <= 8, or for B >= 16 the packed partial sum
// P = {sum over word w, sum over word w + 2} (tree levels up to 8 elements).
template <int B, bool FOLD, bool WANT_SSE>
__device__ __forceinline__ void candidate_wp(const float (&t)[SEG], int w,
                                             const float (&rl)[blocks_per_word<B>()],
                                             const float (&rh)[blocks_per_word<B>()],
                                             const float (&nSl)[blocks_per_word<B>()],
                                             const float (&nSh)[blocks_per_word<B>()], float kf,
                                             uint32_t keep, uint32_t& qa, uint32_t& qb,
                                             float (&el)[blocks_per_word<B>()],
                                             float (&eh)[blocks_per_word<B>()], f32x2& P)
{
    constexpr int G = B < 8 ? B : 8;  // tree width inside one word
    const float z = __uint_as_float(~keep);
    const f32x2 Z = pk2(z, z);
    float ua[8], ub[8];
#if FP4Q_CAND_SCALAR
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = 8 * w + j;
        ua[j] = __fmul_rn(t[i], rl[j / G]);
        ub[j] = __fmul_rn(t[i + 16], rh[j / G]);
    }
#else
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = 8 * w + j;
        upk2(mul2(pk2(t[i], t[i + 16]), pk2(rl[j / G], rh[j / G])), ua[j], ub[j]);
    }
#endif
    qa = e2m1_pack8(ua) & keep;  // see encode_seg on `keep`
    qb = e2m1_pack8(ub) & keep;
#if FP4Q_CAND_SCALAR
    if constexpr (WANT_SSE) {
        float va[8], vb[8], ea[8], eb[8];
        e2m1_unpack8(qa, va);
        e2m1_unpack8(qb, vb);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = 8 * w + j;
            const float ya = FOLD ? __fmul_rn(t[i], kf) : t[i];
            const float yb = FOLD ? __fmul_rn(t[i + 16], kf) : t[i + 16];
            const float da = __fadd_rn(ya, __fmul_rn(va[j], nSl[j / G]));
            const float db = __fadd_rn(yb, __fmul_rn(vb[j], nSh[j / G]));
            ea[j] = __fmul_rn(da, da);
            eb[j] = __fmul_rn(db, db);
        }
#pragma unroll
        for (int h = 1; h < G; h <<= 1)
#pragma unroll
            for (int j = 0; j + h < 8; j += 2 * h) {
                ea[j] = __fadd_rn(ea[j], ea[j + h]);
                eb[j] = __fadd_rn(eb[j], eb[j + h]);
            }
        if constexpr (B <= 8) {
#pragma unroll
            for (int k = 0; k < 8 / B; ++k) {
                el[k] = ea[k * B];
                eh[k] = eb[k * B];
            }
        } else {
            P = pk2(ea[0], eb[0]);
        }
    }
    return;
#endif
    if constexpr (WANT_SSE) {
        float va[8], vb[8];
        e2m1_unpack8(qa, va);
        e2m1_unpack8(qb, vb);
        f32x2 E[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = 8 * w + j;
            const f32x2 NY = fma2(pk2(va[j], vb[j]), pk2(nSl[j / G], nSh[j / G]), Z);
            const f32x2 T = pk2(t[i], t[i + 16]);
            const f32x2 D = FOLD ? fma2(T, pk2(kf, kf), NY) : add2(T, NY);
            E[j] = fma2(D, D, Z);
        }
#pragma unroll
        for (int h = 1; h < G; h <<= 1)
#pragma unroll
            for (int j = 0; j + h < 8; j += 2 * h)
                E[j] = add2(E[j], E[j + h]);
        if constexpr (B <= 8) {
#pragma unroll
            for (int k = 0; k < 8 / B; ++k)
                upk2(E[k * B], el[k], eh[k]);
        } else {
            P = E[0];
        }
    }
}

template <int B, bool FOLD, bool WANT_SSE>
__device__ __forceinline__ void candidate_seg(const float (&t)[SEG], const float (&r)[SEG / B],
                                              const float (&nS)[SEG / B], float kf, uint32_t keep,
                                              uint32_t (&q)[4], float (&sse)[SEG / B])
{
    constexpr int KB = blocks_per_word<B>();
    f32x2 W[2];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        float rl[KB], rh[KB], nl[KB], nh[KB], el[KB], eh[KB];
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            rl[k] = r[(8 * w + k * B) / B];
            rh[k] = r[(8 * w + 16 + k * B) / B];
            nl[k] = nS[(8 * w + k * B) / B];
            nh[k] = nS[(8 * w + 16 + k * B) / B];
        }
        candidate_wp<B, FOLD, WANT_SSE>(t, w, rl, rh, nl, nh, kf, keep, q[w], q[w + 2], el, eh, W[w]);
        if constexpr (WANT_SSE && B <= 8) {
#pragma unroll
            for (int k = 0; k < KB; ++k) {
                sse[(8 * w + k * B) / B] = el[k];
                sse[(8 * w + 16 + k * B) / B] = eh[k];
            }
        }
    }
    if constexpr (WANT_SSE && B >= 16) {
        const f32x2 P = add2(W[0], W[1]);
        if constexpr (B == 16) {
            upk2(P, sse[0], sse[1]);
        } else {
            float lo, hi;
            upk2(P, lo, hi);
            sse[0] = __fadd_rn(lo, hi);
        }
    }
}

// SSE of one B-wide block yb against value(RNE_E2M1(yb * r)) * S (`keep` as
// in encode_seg). The codes of a zero scale need no masking here: u = y * 0 is a signed zero whose
// value times S = 0 is a signed zero, and y - (+-0) == y.
template <int B>
__device__ __forceinline__ float block_sse(const float* yb, float r, float S, uint32_t keep)
{
    float e[B];
    if constexpr (B >= 8) {
#pragma unroll
        for (int g = 0; g < B / 8; ++g) {
            float u[8], v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                u[j] = __fmul_rn(yb[8 * g + j], r);
            e2m1_unpack8(e2m1_pack8(u) & keep, v);  // see encode_seg on `keep`
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float d = __fsub_rn(yb[8 * g + j], __fmul_rn(v[j], S));
                e[8 * g + j] = __fmul_rn(d, d);
            }
        }
    } else {
        float u[4], v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            u[j] = __fmul_rn(yb[j], r);
        e2m1_unpack4(e2m1_pack4(u) & keep, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float d = __fsub_rn(yb[j], __fmul_rn(v[j], S));
            e[j] = __fmul_rn(d, d);
        }
    }
    return tree_sum<B>(e);
}

// Lower bound on the block SSE of every scale whose reciprocal is <= r: the
// tree sum of fl(y^2) over the elements with fl(|y| * r) <= 0.25 (those
// round to code 0 and contribute exactly fl(y^2)), zeros elsewhere. A larger
// scale has a smaller reciprocal, rounds a superset of elements to zero and,
// since the tree sum of non-negative terms is monotone in every term, has an
// SSE at least this large.
template <int B>
__device__ __forceinline__ float block_zero_lb(const float* yb, float r)
{
    float e[B];
#pragma unroll
    for (int j = 0; j < B; ++j) {
        const float u = __fmul_rn(fabsf(yb[j]), r);
        e[j] = u <= 0.25f ? __fmul_rn(yb[j], yb[j]) : 0.0f;
    }
    return tree_sum<B>(e);
}

// Lower bound on the block SSE of every scale S' <= S (code <= c) when the
// block maximum a saturates at S: if fl(a * r) > 5 it rounds to 6 and its
// error term is fl((a - fl(6 S))^2) <= SSE; a smaller scale also saturates and
// moves fl(6 S') further below a (provided fl(6 S) <= a). Returns -1 when
// these conditions do not hold (no bound).
__device__ __forceinline__ float saturation_lb(float a, float r, float S)
{
    const float y6 = __fmul_rn(6.0f, S);
    if (!(__fmul_rn(a, r) > 5.0f) || !(y6 <= a))
        return -1.0f;
    const float d = __fsub_rn(a, y6);
    return __fmul_rn(d, d);
}

// The FOCUS dequantization scale S_dq of each block of a segment: the
// format's abs-max scale (E8M0 2^(floor(log2 amax) - 2) for MXFP4; E4M3 code
// RNE(amax / (6 s_g)) times s_g for NVFP4) and its scale byte.
template <int B, bool MX>
__device__ __forceinline__ void focus_block_scales(const float (&y)[SEG], float sg, float (&S)[SEG / B],
                                                   uint32_t (&sc)[SEG / B])
{
    constexpr int NB = SEG / B;
    float amax[NB];
    block_amax<B>(y, amax);
    if constexpr (MX) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int e = e8m0_exp(amax[b]);
            sc[b] = (uint32_t)(e + 127);
            S[b] = pow2f(e);
        }
    } else {
        const NvConsts kc = nv_consts(sg);
        float qd[NB], qr[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            qd[b] = kc.den6;
            qr[b] = kc.rden6;
        }
        e4m3_quotient_codes<NB>(amax, qd, qr, kc.fast, sc);
#pragma unroll
        for (int b = 0; b < NB; ++b)
            S[b] = __fmul_rn(e4m3_dec(sc[b]), sg);
    }
}

// ------------------------------------------------------------------ stores

// Writes NK floats of segment s (NK = 32 / granularity) to p + s * NK.
template <int NK>
__device__ __forceinline__ void store_seg_floats(float* p, int64_t s, int nvalid, int gran,
                                                 const float (&v)[NK])
{
    float* o = p + s * NK;
    if (nvalid == SEG) {
        if constexpr (NK >= 4) {
#pragma unroll
            for (int k = 0; k < NK / 4; ++k)
                reinterpret_cast<float4*>(o)[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        } else if constexpr (NK == 2) {
            *reinterpret_cast<float2*>(o) = make_float2(v[0], v[1]);
        } else {
            *o = v[0];
        }
    } else {
#pragma unroll
        for (int k = 0; k < NK; ++k)
            if (k * gran < nvalid)
                o[k] = v[k];
    }
}

// NB = SEG / B bytes (one per block) at p (NB-byte aligned).
template <int NB>
__device__ __forceinline__ void store_bytes(uint8_t* p, const uint32_t (&v)[NB])
{
    if constexpr (NB == 1) {
        *p = (uint8_t)v[0];
    } else if constexpr (NB == 2) {
        *reinterpret_cast<uint16_t*>(p) = (uint16_t)(v[0] | (v[1] << 8));
    } else if constexpr (NB == 4) {
        *reinterpret_cast<uint32_t*>(p) = v[0] | (v[1] << 8) | (v[2] << 16) | (v[3] << 24);
    } else {
        uint2 w;
        w.x = v[0] | (v[1] << 8) | (v[2] << 16) | (v[3] << 24);
        w.y = v[4] | (v[5] << 8) | (v[6] << 16) | (v[7] << 24);
        *reinterpret_cast<uint2*>(p) = w;
    }
}

template <int NB>
__device__ __forceinline__ void store_floats(float* p, const float (&v)[NB])
{
    if constexpr (NB == 1) {
        *p = v[0];
    } else if constexpr (NB == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else if constexpr (NB == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
        reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // RNE, lo in the low half
    return *reinterpret_cast<uint32_t*>(&h);
}

// Writes the 32 values of segment s as fp32 (kind 1) or bf16 (kind 2);
// only the first nvalid elements when the segment is partial.
__device__ __forceinline__ void store_seg_values(void* out, int kind, int64_t s, int nvalid,
                                                 const float (&v)[SEG])
{
    if (kind == 1) {
        float* o = reinterpret_cast<float*>(out) + s * SEG;
        if (nvalid == SEG) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                reinterpret_cast<float4*>(o)[k] =
                    make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < SEG; ++i)
                if (i < nvalid)
                    o[i] = v[i];
        }
    } else if (kind == 2) {
        uint16_t* o = reinterpret_cast<uint16_t*>(out) + s * SEG;
        if (nvalid == SEG) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint4 w;
                w.x = pack_bf16x2(v[8 * k + 0], v[8 * k + 1]);
                w.y = pack_bf16x2(v[8 * k + 2], v[8 * k + 3]);
                w.z = pack_bf16x2(v[8 * k + 4], v[8 * k + 5]);
                w.w = pack_bf16x2(v[8 * k + 6], v[8 * k + 7]);
                reinterpret_cast<uint4*>(o)[k] = w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < SEG; ++i) {
                if (i < nvalid) {
                    __nv_bfloat16 h = __float2bfloat16_rn(v[i]);
                    o[i] = *reinterpret_cast<uint16_t*>(&h);
                }
            }
        }
    }
}

}  // namespace fp4q
