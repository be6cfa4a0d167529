// gptq.cu -- GPTQ error feedback with static groups: the error-feedback part
// of MR-GPTQ ("Bridging the Gap Between Promise and Performance for
// Microscaling FP4 Quantization", 技術概要 §2.2: GPTQ with the MSE-optimised
// grid, static activation reordering and rotations).
//
// The block scales are fixed beforehand (static groups). Columns are taken
// in a processing order perm (the static activation order) against U, the
// upper Cholesky factor of the inverse Hessian in that order. Work proceeds
// in batches of 128 positions ("lazy batch updates"):
//
//   gptq_gather_kernel   work[i][j] = W[i][perm[j]] widened to fp32 (with a
//                        rotation: gptq_rotate_gather_kernel, the row rotated
//                        blockwise first, as the quantizer rotates it)
//   gptq_batch_kernel    one warp per row runs the 128 positions of a batch
//                        in order: quantize with the fixed scale, error
//                        e = (w - value * S) / U[j][j], spread inside the batch
//                        (w_k = fma(-e, U[j][k], w_k)); the codes go to their
//                        original column, e replaces the dead weight in work
//   gptq_trailing_kernel every later column: t = fma chain of e_j * U[j][k]
//                        over the batch (j ascending, from 0), w_k -= t; a
//                        persistent fp32 CUDA-core GEMM without split-K, so
//                        each element's sum has the fixed order
//
// Rows are independent: a row's result depends only on its weights, its
// scales and U. Every floating-point step is one IEEE fp32 operation (fma
// where the definition has one), so the codes equal the oracle's bit for bit.
#include <cuda_fp16.h>

#include "fp4q_device.cuh"
#include "internal.h"

namespace fp4q {
namespace {

constexpr int GB = 128;           // positions per batch
constexpr int ROWS_PER_CTA = 16;  // batch kernel: one warp per row (4096 rows: one wave)
constexpr int TR = 128;           // trailing kernel: 128 rows x 64 columns per CTA
constexpr int TC = 64;
constexpr int TTHREADS = 256;     // 16 x 16 threads, 8 x 4 outputs each

__device__ __forceinline__ int64_t column_of(const GptqArgs& a, int64_t j)
{
    if (a.perm == nullptr)
        return j;
    const int32_t c = a.perm[j];
    if (c < 0 || c >= a.K) {
        atomicAdd(a.err, 1u);  // not a permutation of 0..K-1: recorded, column 0 used
        return 0;
    }
    return c;
}

// Dequantization scale of original column col in row i.
__device__ __forceinline__ float scale_at(const GptqArgs& a, int64_t i, int64_t col)
{
    const uint32_t b = a.scales[i * (a.K / a.block) + col / a.block];
    if (a.fmt == 1)
        return e8m0_dec(b);
    if (a.fmt == 2)
        return ue5m3_dec(b);
    return __fmul_rn(e4m3_dec(b), *a.sg);
}

__global__ void __launch_bounds__(256) gptq_gather_kernel(GptqArgs a)
{
    pdl_begin();
    const int64_t t = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (t >= a.rows * a.K)
        return;
    const int64_t i = t / a.K, j = t - i * a.K;
    a.work[t] = __uint_as_float((uint32_t)a.w[i * a.K + column_of(a, j)] << 16);
}

// MR-GPTQ's rotation in front: one CTA per row. Every thread rotates 32-element
// segments of the row exactly as the quantizer does (rotate_seg: widening,
// butterfly stages in ascending order, the factor k_ROT; 64/128-wide chunks
// span neighbouring lanes, so whole warps take part) into a shared copy of
// the row in original column order, which is then gathered into processing
// order: work[i][j] = rotated(W)[i][perm[j]].
template <int ROT>
__global__ void __launch_bounds__(1024) gptq_rotate_gather_kernel(GptqArgs a)
{
    extern __shared__ float rowbuf[];  // [K]
    pdl_begin();
    const int64_t i = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int64_t nseg = a.K / SEG;
    const int64_t nseg_warps = (nseg + 31) / 32 * 32;  // whole warps per pass
    const uint16_t* wrow = a.w + i * a.K;
    for (int64_t sg = threadIdx.x; sg < nseg_warps; sg += blockDim.x) {
        float y[SEG];
        load_seg_bf16(wrow, a.K, sg, y);  // zeros past the row
        rotate_seg<ROT>(y, lane);
        if (sg < nseg) {
            float4* o = reinterpret_cast<float4*>(rowbuf + sg * SEG);
#pragma unroll
            for (int k = 0; k < SEG / 4; ++k)
                o[k] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
        }
    }
    __syncthreads();
    float* wo = a.work + i * a.K;
    for (int64_t j = threadIdx.x; j < a.K; j += blockDim.x)
        wo[j] = rowbuf[column_of(a, j)];
}

// E2M1 code of u (RNE, saturating, sign kept) and its exact value, one
// element (see e2m1_pack8 for the operand order of the conversions).
__device__ __forceinline__ uint32_t e2m1_code1(float u)
{
    uint32_t r;
    asm("{\n\t.reg .b8 q;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q, %2, %1;\n\t"
        "cvt.u32.u8 %0, q;\n\t}"
        : "=r"(r)
        : "f"(u), "f"(0.0f));
    return r & 0xFu;
}

__device__ __forceinline__ float e2m1_value1(uint32_t q)
{
    uint32_t h;
    const unsigned short t = (unsigned short)q;
    asm("{\n\t.reg .b8 q0, q1;\n\t"
        "mov.b16 {q0, q1}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t}"
        : "=r"(h)
        : "h"(t));
    return h2_to_f2(h).x;
}

// One warp per row; lane l holds positions l, l + 32, l + 64, l + 96 of the
// batch. U's 128 x 128 diagonal block sits in shared memory. The lane that
// owns a position quantizes it and broadcasts the error; the errors (which
// replace the batch's dead weights in work) and the codes are written once
// per lane at the end of the batch.
__global__ void __launch_bounds__(ROWS_PER_CTA * 32) gptq_batch_kernel(GptqArgs a, int64_t b0)
{
    extern __shared__ float us[];  // [GB][GB]
    pdl_begin();
    for (int e = threadIdx.x; e < GB * GB / 4; e += blockDim.x) {
        const int r = e / (GB / 4), c4 = e - r * (GB / 4);
        reinterpret_cast<float4*>(us)[e] =
            *reinterpret_cast<const float4*>(a.U + (b0 + r) * a.K + b0 + 4 * c4);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t i = (int64_t)blockIdx.x * ROWS_PER_CTA + (threadIdx.x >> 5);
    if (i >= a.rows)
        return;  // whole warps
    float* wr = a.work + i * a.K + b0;
    float w[4], S[4], R[4], er[4];
    uint32_t qs[4];
    int64_t col[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int p = lane + 32 * t;
        w[t] = wr[p];
        col[t] = column_of(a, b0 + p);
        S[t] = scale_at(a, i, col[t]);
        R[t] = S[t] == 0.0f ? 0.0f : guarded_rcp(S[t]);
        er[t] = 0.0f;
        qs[t] = 0u;
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll 1
        for (int o = 0; o < 32; ++o) {
            const int jj = 32 * s + o;
            float err = 0.0f;
            if (lane == o) {
                uint32_t q = 0;
                float deq = 0.0f;
                if (S[s] != 0.0f) {
                    q = e2m1_code1(__fmul_rn(w[s], R[s]));
                    deq = __fmul_rn(e2m1_value1(q), S[s]);
                }
                err = __fdiv_rn(__fsub_rn(w[s], deq), us[jj * GB + jj]);
                er[s] = err;
                qs[s] = q;
            }
            err = __shfl_sync(0xFFFFFFFFu, err, o);
            const float* urow = us + jj * GB + lane;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if (t > s || (t == s && lane > o))
                    w[t] = __fmaf_rn(-err, urow[32 * t], w[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        wr[lane + 32 * t] = er[t];
        if (qs[t] != 0) {
            const int64_t e = i * a.K + col[t];
            atomicOr(reinterpret_cast<unsigned*>(a.codes) + (e >> 3), qs[t] << (4u * (uint32_t)(e & 7)));
        }
    }
}

__device__ __forceinline__ void cp_async16(float* smem, const float* gmem)
{
    const unsigned d = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

// work[i][k] -= sum over the batch of e[i][j] * U[b0 + j][k] for k >= b0 + GB,
// each sum an fma chain in j order from 0. Persistent: every CTA takes a
// contiguous run of (row tile, column tile) items, row tile major, so the
// 128 x 128 error tile is loaded once per row tile; the 128 x 64 U tiles
// stream through two shared buffers by asynchronous copies, the next one in
// flight while the current one is used. Each thread accumulates 8 x 4
// outputs (rows 4ty..4ty+3 and 64+4ty.., columns 4tx..4tx+3) from three
// 128-bit shared loads per j; its old weights are fetched before the sums so
// their latency hides behind them.
__global__ void __launch_bounds__(TTHREADS) gptq_trailing_kernel(GptqArgs a, int64_t b0, int64_t items,
                                                                   int64_t col_tiles)
{
    extern __shared__ float sm[];
    float* es = sm;              // [GB][TR]: es[j][r] = e of row r0 + r at position j
    float* ub = sm + GB * TR;    // 2 x [GB][TC]: ut[j][c] = U[b0 + j][k0 + c]
    pdl_begin();
    const int64_t first = (int64_t)blockIdx.x * items / gridDim.x;
    const int64_t last = ((int64_t)blockIdx.x + 1) * items / gridDim.x;
    if (first >= last)
        return;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    auto load_u = [&](int64_t item, int buf) {
        const int64_t k0 = b0 + GB + (item % col_tiles) * TC;
        float* ut = ub + buf * (GB * TC);
        for (int e = threadIdx.x; e < GB * TC / 4; e += TTHREADS) {
            const int jj = e / (TC / 4), c4 = e - jj * (TC / 4);
            cp_async16(ut + 4 * e, a.U + (b0 + jj) * a.K + k0 + 4 * c4);
        }
        cp_async_commit();
    };
    load_u(first, 0);
    int64_t cur_rt = -1;
    int buf = 0;
    for (int64_t it = first; it < last; ++it) {
        const int64_t rt = it / col_tiles;
        const int64_t r0 = rt * TR;
        const int64_t k0 = b0 + GB + (it % col_tiles) * TC;
        if (it + 1 < last) {
            load_u(it + 1, buf ^ 1);
            cp_async_wait<1>();  // this item's U tile has landed (the next may be in flight)
        } else {
            cp_async_wait<0>();
        }
        if (rt != cur_rt) {
            __syncthreads();  // nobody still reads the previous error tile
            for (int e = threadIdx.x; e < TR * GB / 4; e += TTHREADS) {
                const int r = e % TR, j4 = e / TR;
                const int64_t row = r0 + r;
                float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (row < a.rows)
                    v = *reinterpret_cast<const float4*>(a.work + row * a.K + b0 + 4 * j4);
                es[(4 * j4) * TR + r] = v.x;
                es[(4 * j4 + 1) * TR + r] = v.y;
                es[(4 * j4 + 2) * TR + r] = v.z;
                es[(4 * j4 + 3) * TR + r] = v.w;
            }
            cur_rt = rt;
        }
        __syncthreads();  // error tile and this U tile visible to all
        float4 old[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int64_t row = r0 + (r < 4 ? 4 * ty + r : TR / 2 + 4 * ty + r - 4);
            old[r] = row < a.rows ? *reinterpret_cast<const float4*>(a.work + row * a.K + k0 + 4 * tx)
                                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        const float* ut = ub + buf * (GB * TC);
        // acc[p][c] = {sum of row 2p, sum of row 2p + 1} at column c: each lane
        // of the packed fma is the same single-rounding fma as the scalar chain
        f32x2 acc[4][4];
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[p][c] = pk2(0.0f, 0.0f);
#pragma unroll 4
        for (int jj = 0; jj < GB; ++jj) {
            const float4 e0 = reinterpret_cast<const float4*>(es + jj * TR)[ty];
            const float4 e1 = reinterpret_cast<const float4*>(es + jj * TR + TR / 2)[ty];
            const float4 u0 = reinterpret_cast<const float4*>(ut + jj * TC)[tx];
            const f32x2 ep[4] = {pk2(e0.x, e0.y), pk2(e0.z, e0.w), pk2(e1.x, e1.y), pk2(e1.z, e1.w)};
            const f32x2 ud[4] = {pk2(u0.x, u0.x), pk2(u0.y, u0.y), pk2(u0.z, u0.z), pk2(u0.w, u0.w)};
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    acc[p][c] = fma2(ep[p], ud[c], acc[p][c]);
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int64_t row = r0 + (r < 4 ? 4 * ty + r : TR / 2 + 4 * ty + r - 4);
            if (row >= a.rows)
                continue;
            float t[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float lo, hi;
                upk2(acc[r / 2][c], lo, hi);
                t[c] = (r & 1) ? hi : lo;
            }
            float4 v = old[r];
            v.x = __fsub_rn(v.x, t[0]);
            v.y = __fsub_rn(v.y, t[1]);
            v.z = __fsub_rn(v.z, t[2]);
            v.w = __fsub_rn(v.w, t[3]);
            *reinterpret_cast<float4*>(a.work + row * a.K + k0 + 4 * tx) = v;
        }
        __syncthreads();  // this U buffer is free for the copy two items ahead
        buf ^= 1;
    }
}

}  // namespace

cudaError_t launch_gptq(const GptqArgs& a, cudaStream_t st)
{
    if (a.K % GB != 0 || a.rows <= 0 || a.rows * a.K > ((int64_t)1 << 40))
        return cudaErrorInvalidValue;
    const size_t batch_smem = sizeof(float) * GB * GB;
    const size_t trail_smem = sizeof(float) * GB * (TR + 2 * TC);
    cudaError_t e = cudaFuncSetAttribute(gptq_batch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)batch_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gptq_trailing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)trail_smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const int64_t n = a.rows * a.K;
    if (a.rot == 0) {
        e = launch_pdl(gptq_gather_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, a);
    } else {
        const size_t row_smem = sizeof(float) * (size_t)a.K;
        const int64_t nseg_warps = (a.K / SEG + 31) / 32 * 32;
        const unsigned threads = (unsigned)(nseg_warps < 1024 ? nseg_warps : 1024);
        if ((int64_t)row_smem > kGptqRowBytes)
            return cudaErrorInvalidValue;
        auto launch_rot = [&](auto kern) {
            cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)row_smem);
            if (r != cudaSuccess)
                return r;
            return launch_pdl(kern, dim3((unsigned)a.rows), dim3(threads), row_smem, st, a);
        };
        switch (a.rot) {
        case 16: e = launch_rot(gptq_rotate_gather_kernel<16>); break;
        case 32: e = launch_rot(gptq_rotate_gather_kernel<32>); break;
        case 64: e = launch_rot(gptq_rotate_gather_kernel<64>); break;
        case 128: e = launch_rot(gptq_rotate_gather_kernel<128>); break;
        default: e = cudaErrorInvalidValue;
        }
    }
    const unsigned row_ctas = (unsigned)((a.rows + ROWS_PER_CTA - 1) / ROWS_PER_CTA);
    const unsigned row_tiles = (unsigned)((a.rows + TR - 1) / TR);
    for (int64_t b0 = 0; b0 < a.K && e == cudaSuccess; b0 += GB) {
        e = launch_pdl(gptq_batch_kernel, dim3(row_ctas), dim3(ROWS_PER_CTA * 32), batch_smem, st, a, b0);
        const int64_t rest = a.K - b0 - GB;
        if (e == cudaSuccess && rest > 0) {
            const int64_t col_tiles = rest / TC, items = col_tiles * row_tiles;
            const unsigned ctas = (unsigned)(items < sms ? items : sms);  // one per SM
            e = launch_pdl(gptq_trailing_kernel, dim3(ctas), dim3(TTHREADS), trail_smem, st, a, b0, items,
                           col_tiles);
        }
    }
    return e;
}

}  // namespace fp4q
