// aux_kernels.cu -- global abs-max, dequantize, block MSE, FOCUS forward and
// backward, and the element-wise rounding primitives.
//
// Same thread layout as the quantize kernel: one 32-element segment of the
// flattened tensor per thread, 128-bit loads and stores on full segments.
#include <cmath>

#include "fp4q_device.cuh"
#include "internal.h"

namespace fp4q {

constexpr int ATHREADS = 256;
// block MSE and FOCUS forward: 128-thread CTAs measured faster on B200
constexpr int STHREADS = 128;

static inline unsigned grid_for(int64_t nseg, int threads = ATHREADS)
{
    return (unsigned)((nseg + threads - 1) / threads);
}

static inline bool grid_ok(int64_t nseg, int threads = ATHREADS)
{
    const int64_t nblk = (nseg + threads - 1) / threads;
    return nblk > 0 && nblk <= 0x7FFFFFFF;
}

// ------------------------------------------------------------ global abs-max

// Tensor abs-max of the (rotated) tensor, combined across blocks with an
// unsigned atomicMax on the float bits (non-negative floats order like their
// bit patterns). *out must hold +0 before the launch.
template <int ROT>
__global__ void __launch_bounds__(ATHREADS) amax_kernel(const uint16_t* x, int64_t n, unsigned* out)
{
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int64_t nseg = (n + SEG - 1) / SEG;
    const int64_t t = (int64_t)blockIdx.x * ATHREADS + threadIdx.x;
    unsigned m = 0;
    if constexpr (ROT == 0) {
        if (t < nseg) {
            const int64_t base = t * SEG;
            if (base + SEG <= n) {
                const uint4* p = reinterpret_cast<const uint4*>(x + base);
                unsigned acc = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint4 v = ldg_stream(p + k);
                    acc = __vmaxu2(acc, v.x & 0x7FFF7FFFu);
                    acc = __vmaxu2(acc, v.y & 0x7FFF7FFFu);
                    acc = __vmaxu2(acc, v.z & 0x7FFF7FFFu);
                    acc = __vmaxu2(acc, v.w & 0x7FFF7FFFu);
                }
                m = max(acc & 0xFFFFu, acc >> 16) << 16;
            } else {
                for (int64_t i = base; i < n; ++i)
                    m = max(m, ((unsigned)x[i] & 0x7FFFu) << 16);
            }
        }
    } else {
        constexpr int SPT = SegsPerThread<ROT>::value;
        if ((t - lane) * SPT < nseg) {  // warp-uniform
            float y[SPT][SEG];
            load_rotate<ROT>(x, n, t, lane, y);  // past the end reads zeros
#pragma unroll
            for (int k = 0; k < SPT; ++k)
#pragma unroll
                for (int i = 0; i < SEG; ++i)
                    m = max(m, __float_as_uint(fabsf(y[k][i])));
        }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ unsigned wm[ATHREADS / 32];
    if (lane == 0)
        wm[threadIdx.x / 32] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        unsigned v = lane < ATHREADS / 32 ? wm[lane] : 0u;
        v = __reduce_max_sync(0xFFFFFFFFu, v);
        if (lane == 0 && v != 0u)
            atomicMax(out, v);
    }
}

__global__ void finalize_sg_kernel(float* g)
{
    pdl_begin();
    *g = global_scale_of(*g);
}

__global__ void set_one_kernel(float* p)
{
    pdl_begin();
    *p = 1.0f;
}

cudaError_t launch_amax(const uint16_t* x, int64_t n, int rot, unsigned* out, cudaStream_t st)
{
    const int64_t nseg = (n + SEG - 1) / SEG;
    const int64_t nthr = nseg;
    if (!grid_ok(nthr))
        return cudaErrorInvalidValue;
    const unsigned g = grid_for(nthr);
    switch (rot) {
    case 0: return launch_pdl(amax_kernel<0>, dim3(g), dim3(ATHREADS), 0, st, x, n, out);
    case 16: return launch_pdl(amax_kernel<16>, dim3(g), dim3(ATHREADS), 0, st, x, n, out);
    case 32: return launch_pdl(amax_kernel<32>, dim3(g), dim3(ATHREADS), 0, st, x, n, out);
    case 64: return launch_pdl(amax_kernel<64>, dim3(g), dim3(ATHREADS), 0, st, x, n, out);
    case 128: return launch_pdl(amax_kernel<128>, dim3(g), dim3(ATHREADS), 0, st, x, n, out);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_finalize_sg(float* g, cudaStream_t st)
{
    cudaError_t e_ = cudaSuccess;
    e_ = launch_pdl(finalize_sg_kernel, dim3(1), dim3(1), 0, st, g);
    return e_;
}

cudaError_t launch_set_one(float* p, cudaStream_t st)
{
    cudaError_t e_ = cudaSuccess;
    e_ = launch_pdl(set_one_kernel, dim3(1), dim3(1), 0, st, p);
    return e_;
}

// ------------------------------------------------------------ small helpers

// Codes of segment s (16 bytes), byte by byte when the segment is partial.
__device__ __forceinline__ void load_codes(const uint8_t* codes, int64_t s, int nvalid, uint32_t (&q)[4])
{
    if (nvalid == SEG) {
        uint4 c = *reinterpret_cast<const uint4*>(codes + s * (SEG / 2));
        q[0] = c.x; q[1] = c.y; q[2] = c.z; q[3] = c.w;
    } else {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t v = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (2 * (4 * w + k) < nvalid)
                    v |= (uint32_t)codes[s * (SEG / 2) + 4 * w + k] << (8 * k);
            q[w] = v;
        }
    }
}

template <int NB>
__device__ __forceinline__ void load_scale_bytes(const uint8_t* scales, int64_t s, int nvalid, int B,
                                                 uint32_t (&sc)[NB])
{
#pragma unroll
    for (int b = 0; b < NB; ++b)
        sc[b] = (b * B < nvalid) ? (uint32_t)scales[s * NB + b] : 0u;
}

// Block scales from their bytes. FMT: 0 NVFP4 (E4M3 times s_g), 1 MXFP4
// (E8M0), 2 UE5M3 (no global scale).
template <int NB, int FMT>
__device__ __forceinline__ void scales_of(const uint32_t (&sc)[NB], float sg, float (&S)[NB])
{
#pragma unroll
    for (int b = 0; b < NB; ++b)
        S[b] = FMT == 1 ? e8m0_dec(sc[b]) : (FMT == 2 ? ue5m3_dec(sc[b]) : __fmul_rn(e4m3_dec(sc[b]), sg));
}

// ------------------------------------------------------------ dequantize

// Each thread dequantizes DQ_ITEMS groups of EPT consecutive elements (EPT
// = 8 for bf16 output, 4 for fp32): group k of thread (warp w, lane l) starts
// at element ((w * DQ_ITEMS + k) * 32 + l) * EPT, so each load and each
// 16-byte store instruction of a warp covers contiguous memory, and all the
// groups' loads are issued before the first store. A group's elements lie in
// one block unless B = 4 < EPT.
constexpr int DQ_ITEMS = 4;

template <int B, int FMT, int EPT>
__global__ void __launch_bounds__(ATHREADS) dequant_kernel(DequantArgs a)
{
    pdl_begin();
    constexpr int NS = EPT > B ? EPT / B : 1;  // scale bytes per group
    const int64_t t = (int64_t)blockIdx.x * ATHREADS + threadIdx.x;
    const int64_t base = (t >> 5) * (32 * DQ_ITEMS) + (t & 31);  // group index of k = 0
    uint32_t q[DQ_ITEMS], sc[DQ_ITEMS][NS];
#pragma unroll
    for (int k = 0; k < DQ_ITEMS; ++k) {
        const int64_t e0 = (base + 32 * k) * EPT;
        q[k] = 0u;
#pragma unroll
        for (int m = 0; m < NS; ++m)
            sc[k][m] = 0u;
        if (e0 >= a.n)
            continue;
        const int nvalid = (int)min((int64_t)EPT, a.n - e0);  // a multiple of 4
        if (EPT == 8 && nvalid == 8)
            q[k] = *reinterpret_cast<const uint32_t*>(a.codes + e0 / 2);
        else
            q[k] = *reinterpret_cast<const uint16_t*>(a.codes + e0 / 2);
#pragma unroll
        for (int m = 0; m < NS; ++m)
            sc[k][m] = (m * B < nvalid) ? (uint32_t)a.scales[e0 / B + m] : 0u;
    }
    const float sg = FMT == 0 ? *a.sg : 1.0f;
#pragma unroll
    for (int k = 0; k < DQ_ITEMS; ++k) {
        const int64_t e0 = (base + 32 * k) * EPT;
        if (e0 >= a.n)
            break;  // later groups start further on
        const int nvalid = (int)min((int64_t)EPT, a.n - e0);
        float S[NS];
        scales_of<NS, FMT>(sc[k], sg, S);
        float v[EPT];
        if constexpr (EPT == 8)
            e2m1_unpack8(q[k], v);
        else
            e2m1_unpack4(q[k], v);
        float yh[EPT];
#pragma unroll
        for (int j = 0; j < EPT / 2; ++j) {
            const f32x2 Y = mul2(pk2(v[2 * j], v[2 * j + 1]), pk2(S[(2 * j) / B], S[(2 * j + 1) / B]));
            upk2(Y, yh[2 * j], yh[2 * j + 1]);
        }
        if constexpr (EPT == 8) {  // bf16
            uint16_t* o = reinterpret_cast<uint16_t*>(a.out) + e0;
            uint4 w;
            w.x = pack_bf16x2(yh[0], yh[1]);
            w.y = pack_bf16x2(yh[2], yh[3]);
            w.z = pack_bf16x2(yh[4], yh[5]);
            w.w = pack_bf16x2(yh[6], yh[7]);
            if (nvalid == 8)
                *reinterpret_cast<uint4*>(o) = w;
            else
                *reinterpret_cast<uint2*>(o) = make_uint2(w.x, w.y);
        } else {  // fp32
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + e0) =
                make_float4(yh[0], yh[1], yh[2], yh[3]);
        }
    }
}

template <int B, int FMT>
static cudaError_t launch_dequant_b(const DequantArgs& a, cudaStream_t st)
{
    const int ept = a.out_kind == 2 ? 8 : 4;
    const int64_t groups = (a.n + ept - 1) / ept;
    const int64_t nthr = (groups + 32 * DQ_ITEMS - 1) / (32 * DQ_ITEMS) * 32;  // whole warps
    if (!grid_ok(nthr))
        return cudaErrorInvalidValue;
    const unsigned g = grid_for(nthr);
    if (ept == 8)
        return launch_pdl(dequant_kernel<B, FMT, 8>, dim3(g), dim3(ATHREADS), 0, st, a);
    return launch_pdl(dequant_kernel<B, FMT, 4>, dim3(g), dim3(ATHREADS), 0, st, a);
}

template <int FMT>
static cudaError_t launch_dequant_blocks(int block, const DequantArgs& a, cudaStream_t st)
{
    if (FMT == 1 && block != 32)
        return cudaErrorInvalidValue;
    switch (block) {
    case 4: return launch_dequant_b<4, FMT>(a, st);
    case 8: return launch_dequant_b<8, FMT>(a, st);
    case 16: return launch_dequant_b<16, FMT>(a, st);
    case 32: return launch_dequant_b<32, FMT>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_dequant(int fmt, int block, const DequantArgs& a, cudaStream_t st)
{
    switch (fmt) {
    case 0: return launch_dequant_blocks<0>(block, a, st);
    case 1: return launch_dequant_blocks<1>(block, a, st);
    case 2: return launch_dequant_blocks<2>(block, a, st);
    default: return cudaErrorInvalidValue;
    }
}

// Per-warp staging for store_seg_values_warp: 32 lanes' outputs as rows of
// 16-byte chunks (4 for bf16, 8 for fp32) plus one chunk of padding, so that
// neither the row writes nor the transposed reads meet more than two-way bank
// conflicts.
constexpr int kStageChunks = 32 * 9;

// Stores the SEG values of every lane's segment s (fp32 for kind 1, bf16 for
// kind 2; all 32 lanes of the warp call it). A warp of 32 whole segments goes
// through st (the warp's staging area), so that each 16-byte store
// instruction covers 512 contiguous bytes; otherwise each active lane stores
// its own segment.
__device__ __forceinline__ void store_seg_values_warp(void* out, int kind, int64_t s, bool active, int nvalid,
                                                      const float (&v)[SEG], uint4* st)
{
    const int lane = threadIdx.x & 31;
    if (!__all_sync(0xFFFFFFFFu, active && nvalid == SEG)) {
        if (active)
            store_seg_values(out, kind, s, nvalid, v);
        return;
    }
    if (kind == 2) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            st[lane * 5 + k] = make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                                          pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
        __syncwarp();
        uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + (s - lane) * SEG);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int c = 32 * k + lane;
            o[c] = st[(c >> 2) * 5 + (c & 3)];
        }
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            st[lane * 9 + k] = make_uint4(__float_as_uint(v[4 * k]), __float_as_uint(v[4 * k + 1]),
                                          __float_as_uint(v[4 * k + 2]), __float_as_uint(v[4 * k + 3]));
        __syncwarp();
        uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<float*>(out) + (s - lane) * SEG);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int c = 32 * k + lane;
            o[c] = st[(c >> 3) * 9 + (c & 7)];
        }
    }
}

// Dequantize and undo the blockwise rotation: one segment per thread, the
// segment's values decoded, then rotated again by the normalised transform
// (its own inverse; 64/128-wide chunks span neighbouring lanes, so whole warps
// take part). Each decoded product is masked with the run-time all-ones
// `keep` before the butterflies: ptxas would otherwise fuse the packed
// multiply of the decode into the first packed add of the rotation, which
// changes the rounding.
template <int B, int FMT, int ROT>
__global__ void __launch_bounds__(ATHREADS) dequant_rot_kernel(DequantArgs a)
{
    __shared__ uint4 stage[ATHREADS / 32][kStageChunks];
    pdl_begin();
    constexpr int NB = SEG / B;
    const int lane = threadIdx.x & 31;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t s = (int64_t)blockIdx.x * ATHREADS + threadIdx.x;
    if (s - lane >= nseg)  // warp-uniform
        return;
    const bool active = s < nseg;
    const int nvalid = active ? (int)min((int64_t)SEG, a.n - s * SEG) : 0;
    uint32_t q[4] = {0u, 0u, 0u, 0u}, sc[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b)
        sc[b] = 0u;
    if (active) {
        load_codes(a.codes, s, nvalid, q);
        load_scale_bytes<NB>(a.scales, s, nvalid, B, sc);
    }
    const float sg = FMT == 0 ? *a.sg : 1.0f;
    float S[NB], yh[SEG];
    scales_of<NB, FMT>(sc, sg, S);
    decode_seg<B>(q, S, yh);
#pragma unroll
    for (int i = 0; i < SEG; ++i)
        yh[i] = __uint_as_float(__float_as_uint(yh[i]) & a.keep);
    rotate_seg<ROT>(yh, lane);
    store_seg_values_warp(a.out, a.out_kind, s, active, nvalid, yh, stage[threadIdx.x >> 5]);
}

template <int B, int FMT>
static cudaError_t launch_dequant_rot_b(int rot, const DequantArgs& a, cudaStream_t st)
{
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    if (!grid_ok(nseg))
        return cudaErrorInvalidValue;
    const unsigned g = grid_for(nseg);
    switch (rot) {
    case 16: return launch_pdl(dequant_rot_kernel<B, FMT, 16>, dim3(g), dim3(ATHREADS), 0, st, a);
    case 32: return launch_pdl(dequant_rot_kernel<B, FMT, 32>, dim3(g), dim3(ATHREADS), 0, st, a);
    case 64: return launch_pdl(dequant_rot_kernel<B, FMT, 64>, dim3(g), dim3(ATHREADS), 0, st, a);
    case 128: return launch_pdl(dequant_rot_kernel<B, FMT, 128>, dim3(g), dim3(ATHREADS), 0, st, a);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
static cudaError_t launch_dequant_rot_blocks(int block, int rot, const DequantArgs& a, cudaStream_t st)
{
    if (FMT == 1 && block != 32)
        return cudaErrorInvalidValue;
    switch (block) {
    case 4: return launch_dequant_rot_b<4, FMT>(rot, a, st);
    case 8: return launch_dequant_rot_b<8, FMT>(rot, a, st);
    case 16: return launch_dequant_rot_b<16, FMT>(rot, a, st);
    case 32: return launch_dequant_rot_b<32, FMT>(rot, a, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_dequant_rot(int fmt, int block, int rot, const DequantArgs& a, cudaStream_t st)
{
    if (rot == 0)
        return launch_dequant(fmt, block, a, st);
    switch (fmt) {
    case 0: return launch_dequant_rot_blocks<0>(block, rot, a, st);
    case 1: return launch_dequant_rot_blocks<1>(block, rot, a, st);
    case 2: return launch_dequant_rot_blocks<2>(block, rot, a, st);
    default: return cudaErrorInvalidValue;
    }
}

// ------------------------------------------------------------ GEMM alpha

// alpha = s_g(A) * s_g(B) for the NVFP4 GEMM (1 for MXFP4: both NULL).
__global__ void alpha_kernel(const float* sga, const float* sgb, float* alpha)
{
    pdl_begin();
    *alpha = (sga != nullptr && sgb != nullptr) ? __fmul_rn(*sga, *sgb) : 1.0f;
}

cudaError_t launch_alpha(const float* sga, const float* sgb, float* alpha, cudaStream_t st)
{
    return launch_pdl(alpha_kernel, dim3(1), dim3(1), 0, st, sga, sgb, alpha);
}

// ------------------------------------------------------------ block MSE

template <int B, int ROT, int FMT>
__global__ void __launch_bounds__(STHREADS) block_mse_kernel(MseArgs a)
{
    pdl_begin();
    constexpr int NB = SEG / B;
    constexpr int SPT = SegsPerThread<ROT>::value;
    const int lane = threadIdx.x & 31;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t t = (int64_t)blockIdx.x * STHREADS + threadIdx.x;
    if ((t - lane) * SPT >= nseg)
        return;
    float y[SPT][SEG];
    load_rotate<ROT>(a.x, a.n, t, lane, y);
    const float sg = FMT == 0 ? *a.sg : 1.0f;
#pragma unroll
    for (int k = 0; k < SPT; ++k) {
        const int64_t s = t * SPT + k;
        if (s >= nseg)
            continue;
        const int nvalid = (int)min((int64_t)SEG, a.n - s * SEG);
        uint32_t q[4], sc[NB];
        load_codes(a.codes, s, nvalid, q);
        load_scale_bytes<NB>(a.scales, s, nvalid, B, sc);
        float S[NB], sse[NB], m[NB];
        scales_of<NB, FMT>(sc, sg, S);
        sse_seg<B>(y[k], q, S, sse);
#pragma unroll
        for (int b = 0; b < NB; ++b)
            m[b] = __fmul_rn(sse[b], 1.0f / B);
        store_seg_floats<NB>(a.mse, s, nvalid, B, m);
    }
}

template <int B, int FMT>
static cudaError_t launch_mse_rot(int rot, unsigned g, const MseArgs& a, cudaStream_t st)
{
    cudaError_t e_ = cudaSuccess;
    switch (rot) {
    case 0: e_ = launch_pdl(block_mse_kernel<B, 0, FMT>, dim3(g), dim3(STHREADS), 0, st, a); break;
    case 16: e_ = launch_pdl(block_mse_kernel<B, 16, FMT>, dim3(g), dim3(STHREADS), 0, st, a); break;
    case 32: e_ = launch_pdl(block_mse_kernel<B, 32, FMT>, dim3(g), dim3(STHREADS), 0, st, a); break;
    case 64: e_ = launch_pdl(block_mse_kernel<B, 64, FMT>, dim3(g), dim3(STHREADS), 0, st, a); break;
    case 128: e_ = launch_pdl(block_mse_kernel<B, 128, FMT>, dim3(g), dim3(STHREADS), 0, st, a); break;
    default: return cudaErrorInvalidValue;
    }
    return e_;
}

template <int FMT>
static cudaError_t launch_mse_blocks(int block, int rot, unsigned g, const MseArgs& a, cudaStream_t st)
{
    if (FMT == 1 && block != 32)
        return cudaErrorInvalidValue;
    switch (block) {
    case 4: return launch_mse_rot<4, FMT>(rot, g, a, st);
    case 8: return launch_mse_rot<8, FMT>(rot, g, a, st);
    case 16: return launch_mse_rot<16, FMT>(rot, g, a, st);
    case 32: return launch_mse_rot<32, FMT>(rot, g, a, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_block_mse(int fmt, int block, int rot, const MseArgs& a, cudaStream_t st)
{
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t nthr = nseg;
    if (!grid_ok(nthr, STHREADS))
        return cudaErrorInvalidValue;
    const unsigned g = grid_for(nthr, STHREADS);
    switch (fmt) {
    case 0: return launch_mse_blocks<0>(block, rot, g, a, st);
    case 1: return launch_mse_blocks<1>(block, rot, g, a, st);
    case 2: return launch_mse_blocks<2>(block, rot, g, a, st);
    default: return cudaErrorInvalidValue;
    }
}

// ------------------------------------------------------------ FOCUS

// fp16 coefficients of segment s: NK = 32 / SUB values at c + s * NK.
template <int NK>
__device__ __forceinline__ void load_coeffs(const uint16_t* c, int64_t s, int nvalid, int sub, float (&ck)[NK])
{
    const uint16_t* p = c + s * NK;
    if (nvalid == SEG) {
        uint32_t w[NK < 2 ? 1 : NK / 2];
        if constexpr (NK == 1) {
            w[0] = *p;
        } else if constexpr (NK == 2) {
            w[0] = *reinterpret_cast<const uint32_t*>(p);
        } else if constexpr (NK == 4) {
            uint2 v = *reinterpret_cast<const uint2*>(p);
            w[0] = v.x; w[1] = v.y;
        } else {
#pragma unroll
            for (int k = 0; k < NK / 8; ++k) {
                uint4 v = reinterpret_cast<const uint4*>(p)[k];
                w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
            }
        }
        if constexpr (NK == 1) {
            ck[0] = __half2float(__ushort_as_half((unsigned short)w[0]));
        } else {
#pragma unroll
            for (int k = 0; k < NK / 2; ++k) {
                float2 f = h2_to_f2(w[k]);
                ck[2 * k] = f.x;
                ck[2 * k + 1] = f.y;
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < NK; ++k)
            ck[k] = (k * sub < nvalid) ? __half2float(__ushort_as_half(p[k])) : 1.0f;
    }
}

// W_hat = S_dq * Q(W / (S_dq * c_k)), S_dq the format's abs-max block scale.
// (Every thread derives s_g itself: a per-CTA table and barrier, as in the
// quantize kernel, measured slower for this one-segment-per-thread kernel.)
template <int B, int SUB, bool MX>
__global__ void __launch_bounds__(STHREADS) focus_fwd_kernel(FocusFwdArgs a)
{
    __shared__ uint4 stage[STHREADS / 32][kStageChunks];
    pdl_begin();
    constexpr int NB = SEG / B;
    constexpr int NK = SEG / SUB;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t s = (int64_t)blockIdx.x * STHREADS + threadIdx.x;
    const int lane = threadIdx.x & 31;
    float sg = 1.0f;
    if constexpr (!MX) {
        sg = global_scale_of(*a.amax);
        if (a.sg_out != nullptr && s == 0)
            *a.sg_out = sg;
    }
    if (s - lane >= nseg)  // warp-uniform: the warp's stores are staged together
        return;
    const bool active = s < nseg;  // an inactive lane loads nothing (zeros) and stores nothing
    const int nvalid = active ? (int)min((int64_t)SEG, a.n - s * SEG) : 0;
    float y[SEG], ck[NK];
    load_seg_bf16(a.w, a.n, s, y);
    load_coeffs<NK>(a.c, s, nvalid, SUB, ck);

    float S[NB];
    uint32_t sc[NB];
    bool zb[NB];
    focus_block_scales<B, MX>(y, sg, S, sc);
#pragma unroll
    for (int b = 0; b < NB; ++b)
        zb[b] = (S[b] == 0.0f);
    float r[NK];
    bool zk[NK];
#pragma unroll
    for (int k = 0; k < NK; ++k) {
        const int b = (k * SUB) / B;
        zk[k] = zb[b];
        r[k] = zb[b] ? 0.0f : guarded_rcp(__fmul_rn(S[b], ck[k]));
    }
    uint32_t q[4];
    encode_seg<SUB, true>(y, r, zk, a.keep, q);  // packed: measured faster here
    float yh[SEG];
    decode_seg<B>(q, S, yh);
    store_seg_values_warp(a.w_hat, a.out_kind, s, active, nvalid, yh, stage[threadIdx.x >> 5]);
    if (a.codes != nullptr && active) {
        if (nvalid == SEG) {
            *reinterpret_cast<uint4*>(a.codes + s * (SEG / 2)) = make_uint4(q[0], q[1], q[2], q[3]);
            store_bytes<NB>(a.scales + s * NB, sc);
        } else {
#pragma unroll
            for (int i = 0; i < SEG / 2; ++i)
                if (2 * i < nvalid)
                    a.codes[s * (SEG / 2) + i] = (uint8_t)(q[i / 4] >> (8 * (i % 4)));
#pragma unroll
            for (int b = 0; b < NB; ++b)
                if (b * B < nvalid)
                    a.scales[s * NB + b] = (uint8_t)sc[b];
        }
    }
}

template <int B, int SUB, bool MX>
static bool try_ffwd(int sub, unsigned g, const FocusFwdArgs& a, cudaStream_t st, cudaError_t& e)
{
    if constexpr (SUB <= B) {
        if (sub == SUB) {
            e = launch_pdl(focus_fwd_kernel<B, SUB, MX>, dim3(g), dim3(STHREADS), 0, st, a);
            return true;
        }
    }
    return false;
}

template <int B, bool MX>
static cudaError_t launch_ffwd_sub(int sub, unsigned g, const FocusFwdArgs& a, cudaStream_t st)
{
    cudaError_t e = cudaErrorInvalidValue;
    if (try_ffwd<B, 2, MX>(sub, g, a, st, e) || try_ffwd<B, 4, MX>(sub, g, a, st, e) ||
        try_ffwd<B, 8, MX>(sub, g, a, st, e) || try_ffwd<B, 16, MX>(sub, g, a, st, e) ||
        try_ffwd<B, 32, MX>(sub, g, a, st, e))
        return e;
    return cudaErrorInvalidValue;
}

cudaError_t launch_focus_fwd(int mx, int block, int sub, const FocusFwdArgs& a, cudaStream_t st)
{
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    if (!grid_ok(nseg, STHREADS) || sub > block)
        return cudaErrorInvalidValue;
    const unsigned g = grid_for(nseg, STHREADS);
    if (mx)
        return block == 32 ? launch_ffwd_sub<32, true>(sub, g, a, st) : cudaErrorInvalidValue;
    switch (block) {
    case 4: return launch_ffwd_sub<4, false>(sub, g, a, st);
    case 8: return launch_ffwd_sub<8, false>(sub, g, a, st);
    case 16: return launch_ffwd_sub<16, false>(sub, g, a, st);
    case 32: return launch_ffwd_sub<32, false>(sub, g, a, st);
    default: return cudaErrorInvalidValue;
    }
}

// dL/dc_k = -(tree_sum over sub-block k of g * W) / (c_k * c_k).
template <int SUB>
__global__ void __launch_bounds__(ATHREADS) focus_bwd_kernel(FocusBwdArgs a)
{
    pdl_begin();
    constexpr int NK = SEG / SUB;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    const int64_t s = (int64_t)blockIdx.x * ATHREADS + threadIdx.x;
    if (s >= nseg)
        return;
    const int nvalid = (int)min((int64_t)SEG, a.n - s * SEG);
    float w[SEG], g[SEG], ck[NK], dc[NK];
    load_seg_bf16(a.w, a.n, s, w);
    load_seg_bf16(a.g, a.n, s, g);
    load_coeffs<NK>(a.c, s, nvalid, SUB, ck);
#pragma unroll
    for (int i = 0; i < SEG; ++i)
        w[i] = __fmul_rn(g[i], w[i]);
#pragma unroll
    for (int k = 0; k < NK; ++k) {
        const float acc = tree_sum<SUB>(w + k * SUB);
        const float cc = __fmul_rn(ck[k], ck[k]);
        dc[k] = -__fdiv_rn(acc, cc);
    }
    store_seg_floats<NK>(a.dc, s, nvalid, SUB, dc);
}

cudaError_t launch_focus_bwd(int sub, const FocusBwdArgs& a, cudaStream_t st)
{
    cudaError_t e_ = cudaSuccess;
    const int64_t nseg = (a.n + SEG - 1) / SEG;
    if (!grid_ok(nseg))
        return cudaErrorInvalidValue;
    const unsigned g = grid_for(nseg);
    switch (sub) {
    case 2: e_ = launch_pdl(focus_bwd_kernel<2>, dim3(g), dim3(ATHREADS), 0, st, a); break;
    case 4: e_ = launch_pdl(focus_bwd_kernel<4>, dim3(g), dim3(ATHREADS), 0, st, a); break;
    case 8: e_ = launch_pdl(focus_bwd_kernel<8>, dim3(g), dim3(ATHREADS), 0, st, a); break;
    case 16: e_ = launch_pdl(focus_bwd_kernel<16>, dim3(g), dim3(ATHREADS), 0, st, a); break;
    case 32: e_ = launch_pdl(focus_bwd_kernel<32>, dim3(g), dim3(ATHREADS), 0, st, a); break;
    default: return cudaErrorInvalidValue;
    }
    return e_;
}

// ------------------------------------------------------------ primitives

__global__ void e2m1_encode_kernel(const float* u, int64_t n, uint8_t* out)
{
    pdl_begin();
    const int64_t i = (int64_t)blockIdx.x * ATHREADS + threadIdx.x;
    if (i >= n)
        return;
    float t[4] = {u[i], 0.0f, 0.0f, 0.0f};
    out[i] = (uint8_t)(e2m1_pack4(t) & 0xFu);
}

__global__ void e4m3_encode_kernel(const float* v, int64_t n, uint8_t* out)
{
    pdl_begin();
    const int64_t i = (int64_t)blockIdx.x * ATHREADS + threadIdx.x;
    if (i >= n)
        return;
    out[i] = (uint8_t)e4m3_enc(v[i]);
}

cudaError_t launch_e2m1_encode(const float* u, int64_t n, uint8_t* out, cudaStream_t st)
{
    cudaError_t e_ = cudaSuccess;
    if (!grid_ok(n))
        return cudaErrorInvalidValue;
    e_ = launch_pdl(e2m1_encode_kernel, dim3(grid_for(n)), dim3(ATHREADS), 0, st, u, n, out);
    return e_;
}

cudaError_t launch_e4m3_encode(const float* v, int64_t n, uint8_t* out, cudaStream_t st)
{
    cudaError_t e_ = cudaSuccess;
    if (!grid_ok(n))
        return cudaErrorInvalidValue;
    e_ = launch_pdl(e4m3_encode_kernel, dim3(grid_for(n)), dim3(ATHREADS), 0, st, v, n, out);
    return e_;
}

}  // namespace fp4q
