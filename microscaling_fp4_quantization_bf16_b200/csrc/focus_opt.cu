// FOCUS coefficient calibration ("FOCUS: FP4 Optimization via Coupled-Relaxation
// and Dual-Granularity Scaling", Metodologia §1-§3): the coefficients c_k are
// learned by gradient descent through the straight-through estimator.
//
//   focus_update_kernel  g (external) -> dc -> optimizer step on c
//   focus_step_kernel    W -> W_hat (forward) -> g = 2 (W_hat - W) -> dc -> step
//
// One thread per 32-element segment, as the other FOCUS kernels; a segment
// holds 32 / sub whole sub-blocks, so each thread owns its coefficients and
// their optimizer state outright (no reduction across threads, no atomics).
// The master coefficients and the Adam moments are fp32; the forward and the
// gradient use fp16(c), the type the pages give the coefficient.
#include <cuda_fp16.h>

#include "fp4q_device.cuh"
#include "internal.h"

namespace fp4q {
namespace {

constexpr int OTHREADS = 128;

// NK fp32 values of segment s at p + s * NK (NK = 32 / sub); sub-blocks past
// nvalid read as 0.
template <int NK>
__device__ __forceinline__ void load_seg_coef(const float* p, int64_t s, int nvalid, int gran, float (&v)[NK])
{
    const float* q = p + s * NK;
    if (nvalid == SEG) {
        if constexpr (NK >= 4) {
#pragma unroll
            for (int k = 0; k < NK / 4; ++k) {
                const float4 f = reinterpret_cast<const float4*>(q)[k];
                v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
            }
        } else if constexpr (NK == 2) {
            const float2 f = *reinterpret_cast<const float2*>(q);
            v[0] = f.x; v[1] = f.y;
        } else {
            v[0] = *q;
        }
    } else {
#pragma unroll
        for (int k = 0; k < NK; ++k)
            v[k] = (k * gran < nvalid) ? q[k] : 0.0f;
    }
}

// NK fp16 bit patterns of segment s at p + s * NK.
template <int NK>
__device__ __forceinline__ void store_seg_halves(uint16_t* p, int64_t s, int nvalid, int gran,
                                                 const uint32_t (&h)[NK])
{
    uint16_t* o = p + s * NK;
    if (nvalid == SEG) {
        if constexpr (NK >= 8) {
#pragma unroll
            for (int k = 0; k < NK / 8; ++k)
                reinterpret_cast<uint4*>(o)[k] =
                    make_uint4(h[8 * k] | (h[8 * k + 1] << 16), h[8 * k + 2] | (h[8 * k + 3] << 16),
                               h[8 * k + 4] | (h[8 * k + 5] << 16), h[8 * k + 6] | (h[8 * k + 7] << 16));
        } else if constexpr (NK == 4) {
            *reinterpret_cast<uint2*>(o) = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
        } else if constexpr (NK == 2) {
            *reinterpret_cast<uint32_t*>(o) = h[0] | (h[1] << 16);
        } else {
            *o = (uint16_t)h[0];
        }
    } else {
#pragma unroll
        for (int k = 0; k < NK; ++k)
            if (k * gran < nvalid)
                o[k] = (uint16_t)h[k];
    }
}

__device__ __forceinline__ void prefetch_l2(const float* p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// fp32 -> fp16 (round to nearest even) -> fp32: the coefficient the forward uses.
__device__ __forceinline__ float coef_used(float c)
{
    return __half2float(__float2half_rn(c));
}

// One optimizer step on a master coefficient; every operation is one IEEE
// fp32 operation with round-to-nearest-even (explicit intrinsics: nothing is
// contracted). Adam in the efficient ordering Kingma & Ba give beside their
// algorithm: the bias corrections are folded into the step size o.alpha.
template <bool ADAM>
__device__ __forceinline__ void opt_step(float dc, const OptConsts& o, float& c, float& m, float& v)
{
    if constexpr (!ADAM) {
        c = __fsub_rn(c, __fmul_rn(o.lr, dc));
    } else {
        m = __fadd_rn(__fmul_rn(o.b1, m), __fmul_rn(o.om1, dc));
        v = __fadd_rn(__fmul_rn(o.b2, v), __fmul_rn(o.om2, __fmul_rn(dc, dc)));
        const float den = __fadd_rn(__fsqrt_rn(v), o.eps);
        c = __fsub_rn(c, __fmul_rn(o.alpha, __fdiv_rn(m, den)));
    }
}

// dc of every sub-block of the segment from its tree sum of g * W (acc[k]),
// then the optimizer step, then the stores of c (and m, v, fp16(c)).
template <int SUB, bool ADAM, int NA>
__device__ __forceinline__ void update_sums(const float (&acc)[NA], const float (&ck)[SEG / SUB], float (&c)[SEG / SUB],
                                            float (&m)[SEG / SUB], float (&v)[SEG / SUB], const OptConsts& o,
                                            float* cp, uint16_t* chp, float* mp, float* vp, int64_t s, int nvalid)
{
    constexpr int NK = SEG / SUB;
    static_assert(NA >= NK, "one sum per sub-block");
    uint32_t h[NK];
#pragma unroll
    for (int k = 0; k < NK; ++k) {
        const float dc = -__fdiv_rn(acc[k], __fmul_rn(ck[k], ck[k]));
        opt_step<ADAM>(dc, o, c[k], m[k], v[k]);
        h[k] = __half_as_ushort(__float2half_rn(c[k]));
    }
    store_seg_floats<NK>(cp, s, nvalid, SUB, c);
    if constexpr (ADAM) {
        store_seg_floats<NK>(mp, s, nvalid, SUB, m);
        store_seg_floats<NK>(vp, s, nvalid, SUB, v);
    }
    if (chp != nullptr)
        store_seg_halves<NK>(chp, s, nvalid, SUB, h);
}

template <int SUB, bool ADAM>
__global__ void __launch_bounds__(OTHREADS) focus_update_kernel(FocusUpdateArgs a)
{
    pdl_begin();
    constexpr int NK = SEG / SUB;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t s = (int64_t)blockIdx.x * OTHREADS + threadIdx.x;
    if (s >= nseg)
        return;
    const int nvalid = (int)min((int64_t)SEG, a.n - s * SEG);
    float w[SEG], g[SEG], c[NK], ck[NK], m[NK], v[NK];
    load_seg_bf16(a.w, a.n, s, w);
    load_seg_bf16(a.g, a.n, s, g);
    load_seg_coef<NK>(a.c, s, nvalid, SUB, c);
    if constexpr (ADAM) {
        load_seg_coef<NK>(a.m, s, nvalid, SUB, m);
        load_seg_coef<NK>(a.v, s, nvalid, SUB, v);
    }
#pragma unroll
    for (int k = 0; k < NK; ++k)
        ck[k] = coef_used(c[k]);
#pragma unroll
    for (int i = 0; i < SEG; ++i)
        w[i] = __fmul_rn(g[i], w[i]);
    float acc[NK];
#pragma unroll
    for (int k = 0; k < NK; ++k)
        acc[k] = tree_sum<SUB>(w + k * SUB);
    update_sums<SUB, ADAM>(acc, ck, c, m, v, a.o, a.c, a.c_half, a.m, a.v, s, nvalid);
}

// Resident CTAs the step kernel is compiled for. With sub-blocks of 8 or more
// it is held to 64 registers (8 CTAs, 32 warps per SM; a few bytes spill):
// measured 8% faster than its unconstrained 80 registers on the 4096 x 4096
// NVFP4 B16 sub-8 step. Smaller sub-blocks keep more per-thread state.
template <int SUB>
constexpr int step_min_blocks() { return SUB >= 8 ? 8 : (SUB == 4 ? 6 : 4); }

// Fused step on L = sum (W_hat - W)^2: the forward is fp4q_focus_fwd's
// (S_dq = the format's abs-max block scale, u = W * (1 / (S_dq * c16)),
// E2M1 RNE, W_hat = val * S_dq), then d = W_hat - W, g = d + d, p = g * W.
template <int B, int SUB, bool MX, bool ADAM>
__global__ void __launch_bounds__(OTHREADS, step_min_blocks<SUB>()) focus_step_kernel(FocusStepArgs a)
{
    pdl_begin();
    constexpr int NB = SEG / B;
    constexpr int NK = SEG / SUB;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t s = (int64_t)blockIdx.x * OTHREADS + threadIdx.x;
    float sg = 1.0f;
    if constexpr (!MX) {
        sg = global_scale_of(*a.amax);
        if (a.sg_out != nullptr && s == 0)
            *a.sg_out = sg;
    }
    if (s >= nseg)
        return;
    const int nvalid = (int)min((int64_t)SEG, a.n - s * SEG);
    float y[SEG], c[NK], ck[NK], m[NK], v[NK];
    load_seg_bf16(a.w, a.n, s, y);
    load_seg_coef<NK>(a.c, s, nvalid, SUB, c);
    if constexpr (ADAM) {
        // the moments are needed only at the end: start their lines towards
        // L2 now, load them into registers after the forward pass
        prefetch_l2(a.m + s * NK);
        prefetch_l2(a.v + s * NK);
    }
    float S[NB];
    uint32_t sc[NB];
    focus_block_scales<B, MX>(y, sg, S, sc);
    float r[NK];
    bool zk[NK];
#pragma unroll
    for (int k = 0; k < NK; ++k) {
        const int b = (k * SUB) / B;
        ck[k] = coef_used(c[k]);
        zk[k] = (S[b] == 0.0f);
        r[k] = zk[k] ? 0.0f : guarded_rcp(__fmul_rn(S[b], ck[k]));
    }
    uint32_t q[4];
    encode_seg<SUB, true>(y, r, zk, a.keep, q);
    // Word by word (8 elements): W_hat = val * S_dq, d = W_hat - W, the
    // products g * W = (d + d) * W in place of W, and d * d; each is
    // tree-summed over groups of G = min(sub, 8) at once. The adjacent-pair
    // tree of a sub-block finishes its groups first, so the group sums are then
    // combined by the same tree: the sums equal tree_sum over the sub-block.
    constexpr int G = SUB < 8 ? SUB : 8;
    constexpr int NG = SEG / G;
    const bool want_sse = a.sse != nullptr;
    float pg[NG], eg[NG];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        float v[8], e[8];
        e2m1_unpack8(q[w], v);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = 8 * w + j;
            const float d = __fsub_rn(__fmul_rn(v[j], S[i / B]), y[i]);
            y[i] = __fmul_rn(__fadd_rn(d, d), y[i]);
            e[j] = __fmul_rn(d, d);
        }
#pragma unroll
        for (int h = 0; h < 8 / G; ++h) {
            pg[w * (8 / G) + h] = tree_sum<G>(y + 8 * w + h * G);
            if (want_sse)
                eg[w * (8 / G) + h] = tree_sum<G>(e + h * G);
        }
    }
    if constexpr (SUB > 8) {
#pragma unroll
        for (int k = 0; k < NK; ++k) {
            pg[k] = tree_sum<SUB / 8>(pg + k * (SUB / 8));
            if (want_sse)
                eg[k] = tree_sum<SUB / 8>(eg + k * (SUB / 8));
        }
    }
    if (want_sse) {
        float es[NK];
#pragma unroll
        for (int k = 0; k < NK; ++k)
            es[k] = eg[k];
        store_seg_floats<NK>(a.sse, s, nvalid, SUB, es);
    }
    if constexpr (ADAM) {
        load_seg_coef<NK>(a.m, s, nvalid, SUB, m);
        load_seg_coef<NK>(a.v, s, nvalid, SUB, v);
    }
    update_sums<SUB, ADAM>(pg, ck, c, m, v, a.o, a.c, a.c_half, a.m, a.v, s, nvalid);
}

unsigned grid_of(int64_t n)
{
    return (unsigned)(((n + SEG - 1) / SEG + OTHREADS - 1) / OTHREADS);
}

bool grid_fits(int64_t n)
{
    return ((n + SEG - 1) / SEG + OTHREADS - 1) / OTHREADS <= (int64_t)0x7FFFFFFF;
}

template <int SUB>
cudaError_t launch_update_sub(bool adam, const FocusUpdateArgs& a, cudaStream_t st)
{
    const dim3 g(grid_of(a.n)), b(OTHREADS);
    return adam ? launch_pdl(focus_update_kernel<SUB, true>, g, b, 0, st, a)
                : launch_pdl(focus_update_kernel<SUB, false>, g, b, 0, st, a);
}

template <int B, int SUB, bool MX>
bool try_step(int sub, bool adam, const FocusStepArgs& a, cudaStream_t st, cudaError_t& e)
{
    if constexpr (SUB <= B) {
        if (sub == SUB) {
            const dim3 g(grid_of(a.n)), b(OTHREADS);
            e = adam ? launch_pdl(focus_step_kernel<B, SUB, MX, true>, g, b, 0, st, a)
                     : launch_pdl(focus_step_kernel<B, SUB, MX, false>, g, b, 0, st, a);
            return true;
        }
    }
    return false;
}

template <int B, bool MX>
cudaError_t launch_step_sub(int sub, bool adam, const FocusStepArgs& a, cudaStream_t st)
{
    cudaError_t e = cudaErrorInvalidValue;
    if (try_step<B, 2, MX>(sub, adam, a, st, e) || try_step<B, 4, MX>(sub, adam, a, st, e) ||
        try_step<B, 8, MX>(sub, adam, a, st, e) || try_step<B, 16, MX>(sub, adam, a, st, e) ||
        try_step<B, 32, MX>(sub, adam, a, st, e))
        return e;
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_focus_update(int sub, bool adam, const FocusUpdateArgs& a, cudaStream_t st)
{
    if (!grid_fits(a.n))
        return cudaErrorInvalidValue;
    switch (sub) {
    case 2: return launch_update_sub<2>(adam, a, st);
    case 4: return launch_update_sub<4>(adam, a, st);
    case 8: return launch_update_sub<8>(adam, a, st);
    case 16: return launch_update_sub<16>(adam, a, st);
    case 32: return launch_update_sub<32>(adam, a, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_focus_step(int mx, int block, int sub, bool adam, const FocusStepArgs& a,
                              cudaStream_t st)
{
    if (!grid_fits(a.n) || sub > block)
        return cudaErrorInvalidValue;
    if (mx)
        return block == 32 ? launch_step_sub<32, true>(sub, adam, a, st) : cudaErrorInvalidValue;
    switch (block) {
    case 4: return launch_step_sub<4, false>(sub, adam, a, st);
    case 8: return launch_step_sub<8, false>(sub, adam, a, st);
    case 16: return launch_step_sub<16, false>(sub, adam, a, st);
    case 32: return launch_step_sub<32, false>(sub, adam, a, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace fp4q
