// quant_kernel.cuh -- the fused rotate -> scale -> encode -> pack kernel.
//
// One thread owns one 32-element segment of the flattened tensor (blocks and
// rotation chunks never straddle rows because cols is a multiple of both).
// The segment is read once with four 128-bit loads, rotated in registers,
// scaled, encoded and packed; the 16 code bytes leave in one 128-bit store.
//
// Scale selection ("Finer is Better (with the Right Scaling)", 手法 2):
//   abs-max      c = RNE_E4M3(amax / (6 s_g))
//   prevent-zero c = max(abs-max code, 0x01)
//   4-over-6     targets 6 and 4; target 4 is kept only if its block SSE is
//                strictly lower
//   brute force  every code 0x01..0x7E, strictly lower SSE wins (ties keep
//                the lower code)
// MXFP4 ("Bridging the Gap ...", 技術概要 §1): S = 2^(floor(log2 amax) - 2).
// UE5M3 scales (the wide-exponent format "Finer is Better ..." compares with
// E4M3 + hierarchical scaling, 意義と主張): the same four strategies over the
// codes of the unsigned 5-exponent / 3-mantissa format, with no global scale.
#pragma once

#include "fp4q_device.cuh"
#include "internal.h"

namespace fp4q {

// CTA shape of the direct-load kernel: 128 threads (one segment each). The
// MXFP4 kernels are also asked to fit 10 CTAs (40 warps) per SM, which caps
// them at 48 registers, the NVFP4 ones (brute force aside) 7 CTAs (72
// registers); all measured faster on B200 than 256-thread CTAs at the
// registers the compiler picks unconstrained.
constexpr int QTHREADS = 128;
template <int STRAT>
struct QMinBlocks {
    static constexpr int value =
        STRAT == K_MX ? 10 : (STRAT == K_BRUTE_FORCE || STRAT == K_MX_BRUTE || STRAT == K_UE_BRUTE_FORCE ? 1 : 7);
};

// Per-CTA constants of the NVFP4 kernels, built once by every CTA: the
// dequantization scale S[c] = E4M3(c) * s_g and its reciprocal R[c] (the
// zero-scale convention gives R[0] = 0) for every code c (index 0x7F unused),
// and the scale-selection constants of s_g. UE5M3 kernels: S[c] = UE5M3(c)
// for c = 0..0xFE (index 0xFF unused).
template <int STRAT>
constexpr int scale_table_size()
{
    return STRAT == K_MX || STRAT == K_MX_BRUTE ? 1 : (is_ue_strat(STRAT) ? 256 : 128);
}

template <int STRAT>
struct ScaleTables {
    float S[scale_table_size<STRAT>()];
    float R[scale_table_size<STRAT>()];
    NvConsts k;
};

// Exact search of one block's scale over the codes 1..MAXC of an increasing
// code -> scale table (E4M3 under s_g, or UE5M3). The candidates from the
// abs-max code c6 - 4 upward are evaluated in ascending order (strictly lower
// SSE wins, so ties keep the lower code); from c6 + 5 on, every third code
// checks block_zero_lb, and once it exceeds the best SSE no larger code can
// win. Codes below c6 - 4 are skipped when saturation_lb at c6 - 5 exceeds the
// best SSE, else searched as well (ties then go to the lower code). A
// non-finite block maximum searches every code in order, as the definition
// does.
template <int B, int MAXC, class Tab>
__device__ __forceinline__ void brute_search(const float* yb, float amax, int c6, const Tab& tab,
                                             uint32_t keep, int& bc_out, float& best_out)
{
    const bool finite = amax <= FLT_MAX;
    const int lo = finite ? max(1, c6 - 4) : 1;
    float best = 0.0f;
    int bc = lo;
#pragma unroll 1
    for (int c = lo; c <= MAXC; ++c) {
        if (finite && c >= c6 + 5 && (c - c6 - 5) % 3 == 0 && block_zero_lb<B>(yb, tab.R[c]) > best)
            break;
        const float v = block_sse<B>(yb, tab.R[c], tab.S[c], keep);
        if (c == lo || v < best) {
            best = v;
            bc = c;
        }
    }
    if (lo > 1 && !(saturation_lb(amax, tab.R[lo - 1], tab.S[lo - 1]) > best)) {
        float bl = 0.0f;
        int cl = 1;
#pragma unroll 1
        for (int c = 1; c < lo; ++c) {
            const float v = block_sse<B>(yb, tab.R[c], tab.S[c], keep);
            if (c == 1 || v < bl) {
                bl = v;
                cl = c;
            }
        }
        if (bl <= best) {
            best = bl;
            bc = cl;
        }
    }
    bc_out = bc;
    best_out = best;
}

// 4-over-6 choice for a whole segment: q, sc, S hold the target-6 result;
// the target-4 candidate (c4, S4, r4, z4) is encoded, both block SSEs are
// computed, and target 4 is kept only where its SSE is strictly lower.
template <int B>
__device__ __forceinline__ void choose_four_over_six(const float (&y)[SEG], uint32_t (&q)[4],
                                                     uint32_t (&sc)[SEG / B], float (&S)[SEG / B],
                                                     float (&sse)[SEG / B], const uint32_t (&c4)[SEG / B],
                                                     const float (&S4)[SEG / B], const float (&r4)[SEG / B],
                                                     const bool (&z4)[SEG / B], uint32_t keep)
{
    constexpr int NB = SEG / B;
    float sse4[NB];
    uint32_t q4w[4];
    encode_seg<B, B == 32>(y, r4, z4, keep, q4w);
    sse_seg<B>(y, q, S, sse);
    sse_seg<B>(y, q4w, S4, sse4);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (sse4[(8 * w + j) / B] < sse[(8 * w + j) / B])
                m |= 0xFu << (4 * j);
        q[w] = (q[w] & ~m) | (q4w[w] & m);
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        if (sse4[b] < sse[b]) {
            sc[b] = c4[b];
            S[b] = S4[b];
            sse[b] = sse4[b];
        }
    }
}

// Scale selection, encoding and stores for one 32-element segment s whose
// (rotated) values are y. nvalid < 32 only for the last segment.
template <int B, int STRAT>
__device__ __forceinline__ void process_segment(const float (&y)[SEG], int64_t s, int nvalid,
                                                const QuantArgs& a, const ScaleTables<STRAT>& tab)
{
    constexpr int NB = SEG / B;
    float amax[NB];
    block_amax<B>(y, amax);

    float S[NB], r[NB], sse[NB];
    bool zero[NB];
    uint32_t sc[NB], q[4];
    bool have_sse = false;

    if constexpr (STRAT == K_MX) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int e = e8m0_exp(amax[b]);
            sc[b] = (uint32_t)(e + 127);
            S[b] = pow2f(e);
            r[b] = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact
            zero[b] = false;
        }
        encode_seg<B, true>(y, r, zero, a.keep, q);  // packed: measured faster here
    } else if constexpr (STRAT == K_MX_BRUTE) {
        // MXFP4 MSE-optimised scale: every E8M0 byte 0..254 (S = 2^(byte -
        // 127)), searched like the NVFP4 brute force below -- upward from the
        // abs-max byte - 1, stopped by block_zero_lb (checked from abs-max + 2),
        // lower bytes skipped under saturation_lb; ties keep the lower byte.
        // (At abs-max - 2 the block maximum is 16 to 32 times the scale, so
        // the saturation bound almost always excludes every lower byte.)
        static_assert(B == 32, "MXFP4 blocks are 32 wide");
        const float am = amax[0];
        const bool finite = am <= FLT_MAX;
        const int babs = e8m0_exp(am) + 127;
        const int lo = finite ? max(0, babs - 1) : 0;
        float best = 0.0f;
        int bb = lo;
#pragma unroll 1
        for (int bt = lo; bt <= 254; ++bt) {
            const float rb = pow2f(127 - bt);
            if (finite && bt >= babs + 2 && block_zero_lb<32>(y, rb) > best)
                break;
            const float v = block_sse<32>(y, rb, pow2f(bt - 127), a.keep);
            if (bt == lo || v < best) {
                best = v;
                bb = bt;
            }
        }
        if (lo > 0 && !(saturation_lb(am, pow2f(128 - lo), pow2f(lo - 128)) > best)) {
            float bl = 0.0f;
            int cl = 0;
#pragma unroll 1
            for (int bt = 0; bt < lo; ++bt) {
                const float v = block_sse<32>(y, pow2f(127 - bt), pow2f(bt - 127), a.keep);
                if (bt == 0 || v < bl) {
                    bl = v;
                    cl = bt;
                }
            }
            if (bl <= best) {
                best = bl;
                bb = cl;
            }
        }
        sc[0] = (uint32_t)bb;
        S[0] = pow2f(bb - 127);
        r[0] = pow2f(127 - bb);
        zero[0] = false;
        sse[0] = best;
        encode_seg<B, true>(y, r, zero, a.keep, q);
        have_sse = true;
    } else if constexpr (STRAT == K_BRUTE_FORCE) {
        // Exact search with pruning (brute_search), from the abs-max code c6.
        const NvConsts k = tab.k;
        float qd[NB], qr[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            qd[b] = k.den6;
            qr[b] = k.rden6;
        }
        uint32_t c6[NB];
        e4m3_quotient_codes<NB>(amax, qd, qr, k.fast, c6);
        static_for<NB>([&](auto bi) {
            constexpr int b = decltype(bi)::value;
            int bc;
            float best;
            brute_search<B, 0x7E>(y + b * B, amax[b], (int)c6[b], tab, a.keep, bc, best);
            sc[b] = (uint32_t)bc;
            S[b] = tab.S[bc];
            r[b] = tab.R[bc];
            zero[b] = (S[b] == 0.0f);
            sse[b] = best;
        });
        encode_seg<B>(y, r, zero, a.keep, q);
        have_sse = true;
    } else if constexpr (is_ue_strat(STRAT)) {
        // UE5M3 scales, no global scale: the candidate code of target T is
        // RNE_UE5M3(amax / T) -- one IEEE division for T = 6; for T = 4 the
        // product by 0.25 is the same correctly rounded quotient.
        uint32_t c6[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b)
            c6[b] = ue5m3_enc(__fdiv_rn(amax[b], 6.0f));
        if constexpr (STRAT == K_UE_BRUTE_FORCE) {
            static_for<NB>([&](auto bi) {
                constexpr int b = decltype(bi)::value;
                int bc;
                float best;
                brute_search<B, 0xFE>(y + b * B, amax[b], (int)c6[b], tab, a.keep, bc, best);
                sc[b] = (uint32_t)bc;
                S[b] = tab.S[bc];
                r[b] = tab.R[bc];
                zero[b] = (S[b] == 0.0f);
                sse[b] = best;
            });
            encode_seg<B>(y, r, zero, a.keep, q);
            have_sse = true;
        } else {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                uint32_t c = c6[b];
                if constexpr (STRAT == K_UE_PREVENT_ZERO)
                    c = max(c, 1u);
                sc[b] = c;
                S[b] = tab.S[c];
                r[b] = tab.R[c];
                zero[b] = (S[b] == 0.0f);
            }
            encode_seg<B, B == 32>(y, r, zero, a.keep, q);
            if constexpr (STRAT == K_UE_FOUR_OVER_SIX) {
                uint32_t c4[NB];
                float S4[NB], r4[NB];
                bool z4[NB];
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    c4[b] = ue5m3_enc(__fmul_rn(amax[b], 0.25f));
                    S4[b] = tab.S[c4[b]];
                    r4[b] = tab.R[c4[b]];
                    z4[b] = (S4[b] == 0.0f);
                }
                choose_four_over_six<B>(y, q, sc, S, sse, c4, S4, r4, z4, a.keep);
                have_sse = true;
            }
        }
    } else if constexpr (STRAT == K_FOUR_OVER_SIX && B <= 8) {
        // 4-over-6 for blocks of 4 or 8, one half segment (words w and w + 2)
        // at a time, so the candidates' temporaries of only half the blocks
        // are live at once. Same operations as the segment form below.
        const NvConsts k = tab.k;
        float qa[2 * NB], qd[2 * NB], qr[2 * NB];
        uint32_t qc[2 * NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            qa[b] = amax[b];
            qd[b] = k.den6;
            qr[b] = k.rden6;
            qa[NB + b] = amax[b];
            qd[NB + b] = k.den4;
            qr[NB + b] = k.rden4;
        }
        e4m3_quotient_codes<2 * NB>(qa, qd, qr, k.fast, qc);
        constexpr int KB = 8 / B;  // blocks per word
        static_for<2>([&](auto wi) {
            constexpr int w = decltype(wi)::value;
            constexpr int bl = 8 * w / B, bh = (8 * w + 16) / B;  // first block of each word
            float S6l[KB], S6h[KB], S4l[KB], S4h[KB], r6l[KB], r6h[KB], r4l[KB], r4h[KB];
            uint32_t z6l = 0, z6h = 0, z4l = 0, z4h = 0;
            constexpr uint32_t BM = B == 4 ? 0xFFFFu : 0xFFFFFFFFu;  // nibbles of one block
#pragma unroll
            for (int t = 0; t < KB; ++t) {
                S6l[t] = tab.S[qc[bl + t]];
                r6l[t] = tab.R[qc[bl + t]];
                S6h[t] = tab.S[qc[bh + t]];
                r6h[t] = tab.R[qc[bh + t]];
                S4l[t] = tab.S[qc[NB + bl + t]];
                r4l[t] = tab.R[qc[NB + bl + t]];
                S4h[t] = tab.S[qc[NB + bh + t]];
                r4h[t] = tab.R[qc[NB + bh + t]];
                z6l |= S6l[t] == 0.0f ? BM << (4 * B * t) : 0u;
                z6h |= S6h[t] == 0.0f ? BM << (4 * B * t) : 0u;
                z4l |= S4l[t] == 0.0f ? BM << (4 * B * t) : 0u;
                z4h |= S4h[t] == 0.0f ? BM << (4 * B * t) : 0u;
            }
            uint32_t q6l, q6h, q4l, q4h;
            encode_word_pair<B>(y, w, r6l, r6h, z6l, z6h, a.keep, q6l, q6h);
            encode_word_pair<B>(y, w, r4l, r4h, z4l, z4h, a.keep, q4l, q4h);
            float e6l[KB], e6h[KB], e4l[KB], e4h[KB];
            sse_word_pair<B>(y, w, q6l, q6h, S6l, S6h, e6l, e6h);
            sse_word_pair<B>(y, w, q4l, q4h, S4l, S4h, e4l, e4h);
            uint32_t ml = 0, mh = 0;
#pragma unroll
            for (int t = 0; t < KB; ++t) {
                const bool fl = e4l[t] < e6l[t], fh = e4h[t] < e6h[t];
                ml |= fl ? BM << (4 * B * t) : 0u;
                mh |= fh ? BM << (4 * B * t) : 0u;
                sc[bl + t] = fl ? qc[NB + bl + t] : qc[bl + t];
                S[bl + t] = fl ? S4l[t] : S6l[t];
                sse[bl + t] = fl ? e4l[t] : e6l[t];
                sc[bh + t] = fh ? qc[NB + bh + t] : qc[bh + t];
                S[bh + t] = fh ? S4h[t] : S6h[t];
                sse[bh + t] = fh ? e4h[t] : e6h[t];
            }
            q[w] = (q6l & ~ml) | (q4l & ml);
            q[w + 2] = (q6h & ~mh) | (q4h & mh);
        });
        have_sse = true;
    } else {
        // Scale codes of the targets in use: 6, and 4 for 4-over-6.
        const NvConsts k = tab.k;
        constexpr bool FOUR = STRAT == K_FOUR_OVER_SIX;
        constexpr int NQ = FOUR ? 2 * NB : NB;
        float qa[NQ], qd[NQ], qr[NQ];
        uint32_t qc[NQ];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            qa[b] = amax[b];
            qd[b] = k.den6;
            qr[b] = k.rden6;
            if constexpr (FOUR) {
                qa[NB + b] = amax[b];
                qd[NB + b] = k.den4;
                qr[NB + b] = k.rden4;
            }
        }
        e4m3_quotient_codes<NQ>(qa, qd, qr, k.fast, qc);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            uint32_t c = qc[b];
            if constexpr (STRAT == K_PREVENT_ZERO)
                c = max(c, 1u);
            sc[b] = c;
            S[b] = tab.S[c];
            r[b] = tab.R[c];
            zero[b] = (S[b] == 0.0f);
        }
        encode_seg<B, B == 32>(y, r, zero, a.keep, q);  // packed measured faster for B = 32 only
        if constexpr (FOUR) {
            float S4[NB], r4[NB];
            bool z4[NB];
            uint32_t c4[NB];
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                c4[b] = qc[NB + b];
                S4[b] = tab.S[c4[b]];
                r4[b] = tab.R[c4[b]];
                z4[b] = (S4[b] == 0.0f);
            }
            choose_four_over_six<B>(y, q, sc, S, sse, c4, S4, r4, z4, a.keep);
            have_sse = true;
        }
    }

    if (a.mse != nullptr && !have_sse)
        sse_seg<B>(y, q, S, sse);

    float m[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b)
        m[b] = __fmul_rn(sse[b], 1.0f / B);  // exact power-of-two division

    if (nvalid == SEG) {
        *reinterpret_cast<uint4*>(a.codes + s * (SEG / 2)) = make_uint4(q[0], q[1], q[2], q[3]);
        if (NB <= 2 && a.mma_spr != 0) {
            // block-scaled MMA layout: 512-byte atoms of 128 rows x 4 blocks (row r
            // at 16 (r % 32) + 4 (r / 32 % 4), block j at + j % 4), atoms along K
            // first. Blocks of 16 or 32 only: the segment's first block is even,
            // so its one or two bytes are adjacent inside one atom row.
            const uint32_t r = (uint32_t)s / a.mma_spr;
            const uint32_t kb = ((uint32_t)s - r * a.mma_spr) * NB;
            const int64_t off = ((int64_t)(r >> 7) * a.mma_atoms_k + (kb >> 2)) * 512 +
                                16 * (r & 31) + 4 * ((r >> 5) & 3) + (kb & 3);
            store_bytes<NB>(a.scales + off, sc);
        } else {
            store_bytes<NB>(a.scales + s * NB, sc);
        }
        if (a.mse != nullptr)
            store_floats<NB>(a.mse + s * NB, m);
    } else {
#pragma unroll
        for (int i = 0; i < SEG / 2; ++i)
            if (2 * i < nvalid)
                a.codes[s * (SEG / 2) + i] = (uint8_t)(q[i / 4] >> (8 * (i % 4)));
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            if (b * B < nvalid) {
                a.scales[s * NB + b] = (uint8_t)sc[b];
                if (a.mse != nullptr)
                    a.mse[s * NB + b] = m[b];
            }
        }
    }
    if (a.dq_kind != 0) {
        float yh[SEG];
        decode_seg<B>(q, S, yh);
        store_seg_values(a.dq, a.dq_kind, s, nvalid, yh);
    }
}

// Builds the CTA's scale tables (NVFP4 kernels; nothing for MXFP4): threads
// 0..127 each compute s_g from the global abs-max and one table entry; thread
// 0 also the scale-selection constants and, in CTA 0, publishes s_g when
// asked. Ends with a CTA barrier.
template <int STRAT>
__device__ __forceinline__ void build_scale_tables(ScaleTables<STRAT>& tab, const QuantArgs& a)
{
    if constexpr (is_ue_strat(STRAT)) {
        for (int c = threadIdx.x; c < 256; c += blockDim.x) {
            const float S = (c <= 0xFE) ? ue5m3_dec((uint32_t)c) : 0.0f;
            tab.S[c] = S;
            tab.R[c] = (S == 0.0f) ? 0.0f : guarded_rcp(S);
        }
        __syncthreads();
    } else if constexpr (STRAT != K_MX && STRAT != K_MX_BRUTE) {
        if (threadIdx.x < 128) {
            const float sg = global_scale_of(*a.amax);
            for (int c = threadIdx.x; c < 128; c += blockDim.x) {
                const float S = (c <= 0x7E) ? __fmul_rn(e4m3_dec((uint32_t)c), sg) : 0.0f;
                tab.S[c] = S;
                tab.R[c] = (S == 0.0f) ? 0.0f : guarded_rcp(S);
            }
            if (threadIdx.x == 0) {
                tab.k = nv_consts(sg);
                if (a.sg_out != nullptr && blockIdx.x == 0)
                    *a.sg_out = sg;
            }
        }
        __syncthreads();
    }
}

// Direct-load kernel: one segment per thread (two for 64/128-wide
// rotations), 128-bit global loads. Used by default, and for the brute-force
// search (compute bound) and flattened lengths that are not a multiple of 64.
template <int B, int ROT, int STRAT>
__global__ void __launch_bounds__(QTHREADS, QMinBlocks<STRAT>::value) quant_kernel(QuantArgs a)
{
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t s = (int64_t)blockIdx.x * QTHREADS + threadIdx.x;
    const bool warp_active = s - lane < nseg;  // warp-uniform

    uint4 raw[4];
    if (warp_active)
        load_seg_raw(a.x, a.n, s, raw);  // in flight while the tables are built
    __shared__ ScaleTables<STRAT> tab;
    build_scale_tables<STRAT>(tab, a);
    if (!warp_active)
        return;

    float y[SEG];
    unpack_seg(raw, y);
    rotate_seg<ROT>(y, lane);  // all 32 lanes take part; past the end holds zeros
    if (s < nseg)
        process_segment<B, STRAT>(y, s, (int)min((int64_t)SEG, a.n - s * SEG), a, tab);
}

template <int B>
cudaError_t launch_quant_impl(int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    const int64_t nseg = (a.n + SEG - 1) / SEG;
#define FP4Q_QCASE(S_, R_)                                                              \
    if (strat == S_ && rot == R_) {                                                     \
        constexpr int64_t per_block = (int64_t)QTHREADS;                     \
        const int64_t nblk = (nseg + per_block - 1) / per_block;                        \
        if (nblk <= 0 || nblk > 0x7FFFFFFF)                                             \
            return cudaErrorInvalidValue;                                               \
        return launch_pdl(quant_kernel<B, R_, S_>, dim3((unsigned)nblk), dim3(QTHREADS), 0, st, a); \
    }
#define FP4Q_QROTS(S_)      \
    FP4Q_QCASE(S_, 0)       \
    FP4Q_QCASE(S_, 16)      \
    FP4Q_QCASE(S_, 32)      \
    FP4Q_QCASE(S_, 64)      \
    FP4Q_QCASE(S_, 128)
    FP4Q_QROTS(K_ABSMAX)
    FP4Q_QROTS(K_PREVENT_ZERO)
    FP4Q_QROTS(K_FOUR_OVER_SIX)
    FP4Q_QROTS(K_BRUTE_FORCE)
    FP4Q_QROTS(K_UE_ABSMAX)
    FP4Q_QROTS(K_UE_PREVENT_ZERO)
    FP4Q_QROTS(K_UE_FOUR_OVER_SIX)
    FP4Q_QROTS(K_UE_BRUTE_FORCE)
    if constexpr (B == 32) {
        FP4Q_QROTS(K_MX)
        FP4Q_QROTS(K_MX_BRUTE)
    }
#undef FP4Q_QROTS
#undef FP4Q_QCASE
    return cudaErrorInvalidValue;
}

}  // namespace fp4q
