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
// MXFP4 kernels are also asked to fit 9 CTAs (36 warps) per SM, which caps
// them at 56 registers (at 10 CTAs they spill and ran 5% slower), the NVFP4
// ones (brute force aside) 7 CTAs (72 registers); all measured faster on B200
// than 256-thread CTAs at the registers the compiler picks unconstrained.
constexpr int QTHREADS = 128;
#ifndef FP4Q_MX_MINB
#define FP4Q_MX_MINB 9
#endif
#ifndef FP4Q_NV_MINB
#define FP4Q_NV_MINB 7
#endif
#ifndef FP4Q_BRUTE_MINB
#define FP4Q_BRUTE_MINB 1
#endif
template <int STRAT>
struct QMinBlocks {
    static constexpr int value =
        STRAT == K_MX ? FP4Q_MX_MINB
                      : (STRAT == K_BRUTE_FORCE || STRAT == K_MX_BRUTE || STRAT == K_UE_BRUTE_FORCE
                             ? FP4Q_BRUTE_MINB
                             : FP4Q_NV_MINB);
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
// does. (Evaluating two codes at once on packed f32x2 lanes gave the same
// results and ran 2-20% slower: the search is bound by its conversions and
// integer work, not its FP32 issue slots.)
template <int B, int MAXC, class Tab>
__device__ __forceinline__ void brute_search(const float* yb, float amax, int c6, const Tab& tab,
                                             uint32_t keep, int& bc_out, float& best_out)
{
    const bool finite = amax <= FLT_MAX;
    const int lo = finite ? max(1, c6 - 4) : 1;
    auto check = [&](int c) { return finite && c >= c6 + 5 && (c - c6 - 5) % 3 == 0; };
    float best = 0.0f;
    int bc = lo;
#pragma unroll 1
    for (int c = lo; c <= MAXC; ++c) {
        if (check(c) && block_zero_lb<B>(yb, tab.R[c]) > best)
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

// Rotations whose factor k = 1/sqrt(n) is a power of two (16: 2^-2, 64:
// 2^-3) are applied unscaled and k is folded into the encode and the error
// (candidate_seg) for the strategies that take that path.
// MXFP4 abs-max folds k for every rotation width: its scale 2^e is a power of
// two, so fl(fl(t k) 2^-e) = fl(t (k 2^-e)) whenever k 2^-e is a normal
// float (a product that underflows rounds to a signed zero code either way);
// that path writes codes only (the SSE needs fl(t k) itself).
template <int ROT, int STRAT>
__host__ __device__ constexpr bool foldable()
{
    return ((ROT == 16 || ROT == 64) &&
            (STRAT == K_ABSMAX || STRAT == K_PREVENT_ZERO || STRAT == K_FOUR_OVER_SIX ||
             STRAT == K_UE_ABSMAX || STRAT == K_UE_PREVENT_ZERO || STRAT == K_UE_FOUR_OVER_SIX)) ||
           (ROT > 0 && STRAT == K_MX);
}

template <int ROT>
__host__ __device__ constexpr float had_k()
{
    if constexpr (ROT == 0)
        return 1.0f;
    else
        return HadK<ROT>::k;
}

// Scale selection, encoding and stores for one 32-element segment s whose
// (rotated) values are y -- before the multiply by k_ROT when
// foldable<ROT, STRAT>() (rotate_seg<ROT, false>). nvalid < 32 only for the
// last segment.
template <int B, int STRAT, int ROT>
__device__ __forceinline__ void process_segment(float (&y)[SEG], int64_t s, int nvalid,
                                                const QuantArgs& a, const ScaleTables<STRAT>& tab)
{
    constexpr int NB = SEG / B;
    constexpr bool FOLDABLE = foldable<ROT, STRAT>();
    float amax[NB];
    block_amax<B>(y, amax);
    if constexpr (FOLDABLE) {
        // max |fl(k t)| = fl(k max |t|): rounding is monotone (exact here anyway)
#pragma unroll
        for (int b = 0; b < NB; ++b)
            amax[b] = __fmul_rn(amax[b], had_k<ROT>());
    }

    float S[NB], r[NB], sse[NB];
    bool zero[NB];
    uint32_t sc[NB], q[4];

    if constexpr (STRAT == K_MX_BRUTE) {
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
    } else if constexpr (STRAT == K_UE_BRUTE_FORCE) {
        // UE5M3 scales, no global scale: the abs-max code is RNE_UE5M3(amax / 6)
        // (one IEEE division), then the exact search.
        uint32_t c6[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b)
            c6[b] = ue5m3_enc(__fdiv_rn(amax[b], 6.0f));
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
    } else {
        // Abs-max, prevent-zero and 4-over-6 (E4M3 under s_g, or UE5M3), and
        // MXFP4 abs-max: the candidate scale code(s) of each block -- target 6,
        // and target 4 for 4-over-6 -- then one fused encode (+ SSE) per
        // candidate (candidate_seg); 4-over-6 keeps target 4 only where its
        // block SSE is strictly lower.
        constexpr bool UE = is_ue_strat(STRAT);
        constexpr bool MX = STRAT == K_MX;
        constexpr bool FOUR = STRAT == K_FOUR_OVER_SIX || STRAT == K_UE_FOUR_OVER_SIX;
        constexpr bool PZ = STRAT == K_PREVENT_ZERO || STRAT == K_UE_PREVENT_ZERO;
        constexpr int NC = FOUR ? 2 : 1;
        uint32_t cc[NC][NB];  // [0]: target 6 (or the E8M0 byte), [1]: target 4
        if constexpr (MX) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
                cc[0][b] = (uint32_t)(e8m0_exp(amax[b]) + 127);
        } else if constexpr (UE) {
            // RNE_UE5M3(amax / T): one IEEE division for T = 6; for T = 4 the
            // product by 0.25 is the same correctly rounded quotient.
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                cc[0][b] = ue5m3_enc(__fdiv_rn(amax[b], 6.0f));
                if constexpr (FOUR)
                    cc[NC - 1][b] = ue5m3_enc(__fmul_rn(amax[b], 0.25f));
            }
        } else {
            const NvConsts k = tab.k;
            float qa[NC * NB], qd[NC * NB], qr[NC * NB];
            uint32_t qc[NC * NB];
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
            e4m3_quotient_codes<NC * NB>(qa, qd, qr, k.fast, qc);
#pragma unroll
            for (int c = 0; c < NC; ++c)
#pragma unroll
                for (int b = 0; b < NB; ++b)
                    cc[c][b] = qc[c * NB + b];
        }
        if constexpr (PZ) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
                cc[0][b] = max(cc[0][b], 1u);
        }
        // scale and reciprocal of candidate code c
        auto scale_of = [&](uint32_t c) -> float { return MX ? pow2f((int)c - 127) : tab.S[c]; };
        auto rcp_of = [&](uint32_t c) -> float {
            return MX ? __uint_as_float((254u - c) << 23) : tab.R[c];  // MXFP4: 2^-e, exact
        };
        const bool want = FOUR || a.mse != nullptr;

        auto run = [&](auto fold_c) {
            constexpr bool FOLD = decltype(fold_c)::value;
            constexpr float kf = FOLD ? had_k<ROT>() : 1.0f;
            if constexpr (B <= 8) {
                // Blocks lie inside words: decide one word pair at a time.
                constexpr int KB = 8 / B;
                static_for<2>([&](auto wi) {
                    constexpr int w = decltype(wi)::value;
                    float rl[NC][KB], rh[NC][KB], nl[NC][KB], nh[NC][KB];
                    float el[NC][KB] = {}, eh[NC][KB] = {};
                    uint32_t qa[NC], qb[NC];
                    f32x2 unused;
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
#pragma unroll
                        for (int k = 0; k < KB; ++k) {
                            const uint32_t cl = cc[c][w * KB + k], ch = cc[c][(w + 2) * KB + k];
                            rl[c][k] = __fmul_rn(rcp_of(cl), kf);
                            rh[c][k] = __fmul_rn(rcp_of(ch), kf);
                            nl[c][k] = -scale_of(cl);
                            nh[c][k] = -scale_of(ch);
                        }
                        if (want)
                            candidate_wp<B, FOLD, true>(y, w, rl[c], rh[c], nl[c], nh[c], kf, a.keep,
                                                        qa[c], qb[c], el[c], eh[c], unused);
                        else
                            candidate_wp<B, FOLD, false>(y, w, rl[c], rh[c], nl[c], nh[c], kf,
                                                         a.keep, qa[c], qb[c], el[c], eh[c], unused);
                    }
                    uint32_t ml = 0, mh = 0, zl = 0, zh = 0;
                    constexpr uint32_t BM = B == 4 ? 0xFFFFu : 0xFFFFFFFFu;  // nibbles of one block
#pragma unroll
                    for (int k = 0; k < KB; ++k) {
                        const bool fl = FOUR && el[NC - 1][k] < el[0][k];
                        const bool fh = FOUR && eh[NC - 1][k] < eh[0][k];
                        const int bl = w * KB + k, bh = (w + 2) * KB + k;
                        sc[bl] = fl ? cc[NC - 1][bl] : cc[0][bl];
                        sc[bh] = fh ? cc[NC - 1][bh] : cc[0][bh];
                        S[bl] = -(fl ? nl[NC - 1][k] : nl[0][k]);
                        S[bh] = -(fh ? nh[NC - 1][k] : nh[0][k]);
                        sse[bl] = fl ? el[NC - 1][k] : el[0][k];
                        sse[bh] = fh ? eh[NC - 1][k] : eh[0][k];
                        ml |= fl ? BM << (4 * B * k) : 0u;
                        mh |= fh ? BM << (4 * B * k) : 0u;
                        zl |= S[bl] == 0.0f ? BM << (4 * B * k) : 0u;
                        zh |= S[bh] == 0.0f ? BM << (4 * B * k) : 0u;
                    }
                    q[w] = ((qa[0] & ~ml) | (qa[NC - 1] & ml)) & ~zl;
                    q[w + 2] = ((qb[0] & ~mh) | (qb[NC - 1] & mh)) & ~zh;
                });
            } else {
                float rr[NC][NB], nS[NC][NB], se[NC][NB] = {};
                uint32_t qc[NC][4];
#pragma unroll
                for (int c = 0; c < NC; ++c) {
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        rr[c][b] = __fmul_rn(rcp_of(cc[c][b]), kf);
                        nS[c][b] = -scale_of(cc[c][b]);
                    }
                    if (want)
                        candidate_seg<B, FOLD, true>(y, rr[c], nS[c], kf, a.keep, qc[c], se[c]);
                    else
                        candidate_seg<B, FOLD, false>(y, rr[c], nS[c], kf, a.keep, qc[c], se[c]);
                }
                bool four[NB];
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    four[b] = FOUR && se[NC - 1][b] < se[0][b];
                    sc[b] = four[b] ? cc[NC - 1][b] : cc[0][b];
                    S[b] = -(four[b] ? nS[NC - 1][b] : nS[0][b]);
                    sse[b] = four[b] ? se[NC - 1][b] : se[0][b];
                }
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t m4 = 0, mz = 0;  // nibbles taken from target 4; of zero scales
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int b = (8 * w + j) / B;
                        if (four[b])
                            m4 |= 0xFu << (4 * j);
                        if (!MX && S[b] == 0.0f)
                            mz |= 0xFu << (4 * j);
                    }
                    q[w] = ((qc[0][w] & ~m4) | (qc[NC - 1][w] & m4)) & ~mz;
                }
            }
        };
        bool fold = false;
        if constexpr (FOLDABLE) {
            if constexpr (MX) {
                fold = a.mse == nullptr;
#pragma unroll
                for (int b = 0; b < NB; ++b)
                    fold = fold && cc[0][b] <= 127 + 122;  // k 2^-e stays normal
            } else {
                fold = UE || tab.k.fold;
            }
            if (!fold)
                scale_seg<ROT>(y);
        }
        if (fold)
            run(std::integral_constant<bool, true>{});
        else
            run(std::integral_constant<bool, false>{});
    }

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
    unpack_seg<!is_mx_strat(STRAT)>(raw, y);
    // all 32 lanes take part; past the end holds zeros
    rotate_seg<ROT, !foldable<ROT, STRAT>()>(y, lane);
    if (s < nseg)
        process_segment<B, STRAT, ROT>(y, s, (int)min((int64_t)SEG, a.n - s * SEG), a, tab);
}

// Persistent form of the direct-load kernel for the one-pass strategies (the
// searches keep quant_kernel: their registers go to the search). A grid of
// resident CTAs walks tiles of QTHREADS segments (tile t covers segments
// t * QTHREADS ..); as soon as a thread has unpacked its segment of the
// current tile it issues the loads of its segment in the next tile into the
// same registers, so their latency overlaps this tile's arithmetic, and each
// CTA builds its scale tables once.
#ifndef FP4Q_PERSIST
#define FP4Q_PERSIST 1
#endif
#ifndef FP4Q_MXP_MINB
#define FP4Q_MXP_MINB 6
#endif
#ifndef FP4Q_NVP_MINB
#define FP4Q_NVP_MINB 5
#endif
template <int STRAT>
struct PMinBlocks {
    static constexpr int value = STRAT == K_MX ? FP4Q_MXP_MINB : FP4Q_NVP_MINB;
};

template <int STRAT>
__host__ __device__ constexpr bool use_persist()
{
    return FP4Q_PERSIST && STRAT != K_BRUTE_FORCE && STRAT != K_MX_BRUTE && STRAT != K_UE_BRUTE_FORCE &&
           STRAT != K_MX;  // measured: MXFP4 runs faster at the one-shot kernel's occupancy
}

template <int B, int ROT, int STRAT>
__global__ void __launch_bounds__(QTHREADS, PMinBlocks<STRAT>::value)
    quant_persist_kernel(QuantArgs a, int64_t ntiles)
{
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int64_t nseg = a.n / SEG;  // every segment is whole (checked by the launcher)
    const int64_t step = (int64_t)gridDim.x * QTHREADS;
    const uint4* x4 = reinterpret_cast<const uint4*>(a.x);
    // segment s's four 128-bit words, or zeros past the end
    auto fetch = [&](int64_t s, uint4 (&raw)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            raw[k] = s < nseg ? ldg_stream(x4 + 4 * s + k) : make_uint4(0u, 0u, 0u, 0u);
    };
    uint4 raw[4];
    int64_t s = (int64_t)blockIdx.x * QTHREADS + threadIdx.x;
    fetch(s, raw);  // in flight while the tables are built
    __shared__ ScaleTables<STRAT> tab;
    build_scale_tables<STRAT>(tab, a);
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, s += step) {
        float y[SEG];
        unpack_seg<!is_mx_strat(STRAT)>(raw, y);
        if (t + gridDim.x < ntiles)
            fetch(s + step, raw);  // next tile's loads overlap this tile's arithmetic
        if (s - lane < nseg) {     // warp-uniform
            // all 32 lanes take part; past the end holds zeros
            rotate_seg<ROT, !foldable<ROT, STRAT>()>(y, lane);
            if (s < nseg)
                process_segment<B, STRAT, ROT>(y, s, SEG, a, tab);
        }
    }
}

// Resident CTAs per SM of a kernel (queried once per process) times the SM
// count of the current device.
template <typename K>
int64_t resident_ctas(K kernel)
{
    static int per_sm = 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    if (per_sm == 0) {
        int v = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, QTHREADS, 0) != cudaSuccess)
            return -1;
        per_sm = v < 1 ? 1 : v;
    }
    return (int64_t)sms * per_sm;
}

template <int B>
cudaError_t launch_quant_impl(int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    const int64_t nseg = (a.n + SEG - 1) / SEG;
#define FP4Q_QCASE(S_, R_)                                                              \
    if (strat == S_ && rot == R_) {                                                     \
        const int64_t nblk = (nseg + QTHREADS - 1) / QTHREADS;                          \
        if (nblk <= 0 || nblk > 0x7FFFFFFF)                                             \
            return cudaErrorInvalidValue;                                               \
        if constexpr (use_persist<S_>()) {                                              \
          if (a.n % SEG == 0) {                                                         \
            const int64_t res = resident_ctas(quant_persist_kernel<B, R_, S_>);         \
            if (res < 0)                                                                \
                return cudaErrorUnknown;                                                \
            const int64_t grid = nblk < res ? nblk : res;                               \
            return launch_pdl(quant_persist_kernel<B, R_, S_>, dim3((unsigned)grid), dim3(QTHREADS), 0, \
                              st, a, nblk);                                             \
          }                                                                             \
        }                                                                               \
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
