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
//   gptq_gather_kernel   work[i][j] = W[i][perm[j]] widened to fp32
//   gptq_batch_kernel    one warp per row runs the 128 positions of a batch
//                        in order: quantize with the fixed scale, error
//                        e = (w - value * S) / U[j][j], spread inside the batch
//                        (w_k = fma(-e, U[j][k], w_k)); the codes go to their
//                        original column, e replaces the dead weight in work
//   gptq_trailing_kernel every later column: t = fma chain of e_j * U[j][k]
//                        over the batch (j ascending, from 0), w_k -= t; an
//                        fp32 CUDA-core GEMM tile without split-K, so each
//                        element's sum has the fixed order
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

// One warp per row; lane l holds positions l, l + 32, l + 64, l + 96 of the
// batch. U's 128 x 128 diagonal block sits in shared memory.
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
    float w[4], S[4], R[4];
    int64_t word[4];
    uint32_t shift[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int p = lane + 32 * t;
        w[t] = wr[p];
        const int64_t col = column_of(a, b0 + p);
        S[t] = scale_at(a, i, col);
        R[t] = S[t] == 0.0f ? 0.0f : guarded_rcp(S[t]);
        const int64_t e = i * a.K + col;
        word[t] = e >> 3;
        shift[t] = 4u * (uint32_t)(e & 7);
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
                    float u[4] = {__fmul_rn(w[s], R[s]), 0.0f, 0.0f, 0.0f};
                    q = e2m1_pack4(u) & 0xFu;
                    float v[4];
                    e2m1_unpack4(q, v);
                    deq = __fmul_rn(v[0], S[s]);
                }
                err = __fdiv_rn(__fsub_rn(w[s], deq), us[jj * GB + jj]);
                if (q != 0)
                    atomicOr(reinterpret_cast<unsigned*>(a.codes) + word[s], q << shift[s]);
                wr[jj] = err;  // the batch's errors replace its dead weights
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
}

// work[i][k] -= sum over the batch of e[i][j] * U[b0 + j][k] for k >= b0 + GB,
// each sum an fma chain in j order from 0. A 128 x 64 output tile per CTA
// (96 KB of shared memory: two CTAs per SM); each thread accumulates 8 x 4
// outputs (rows 4ty..4ty+3 and 64+4ty.., columns 4tx..4tx+3) from three
// 128-bit shared loads per j.
__global__ void __launch_bounds__(TTHREADS) gptq_trailing_kernel(GptqArgs a, int64_t b0)
{
    extern __shared__ float sm[];
    float* es = sm;             // [GB][TR]: es[j][r] = e of row r0 + r at position j
    float* ut = sm + GB * TR;   // [GB][TC]: ut[j][c] = U[b0 + j][k0 + c]
    pdl_begin();
    const int64_t r0 = (int64_t)blockIdx.y * TR;
    const int64_t k0 = b0 + GB + (int64_t)blockIdx.x * TC;
    for (int e = threadIdx.x; e < TR * GB / 4; e += TTHREADS) {
        const int r = e % TR, j4 = e / TR;  // consecutive threads: consecutive rows
        const int64_t row = r0 + r;
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (row < a.rows)
            v = *reinterpret_cast<const float4*>(a.work + row * a.K + b0 + 4 * j4);
        es[(4 * j4) * TR + r] = v.x;
        es[(4 * j4 + 1) * TR + r] = v.y;
        es[(4 * j4 + 2) * TR + r] = v.z;
        es[(4 * j4 + 3) * TR + r] = v.w;
    }
    for (int e = threadIdx.x; e < GB * TC / 4; e += TTHREADS) {
        const int j = e / (TC / 4), c4 = e - j * (TC / 4);
        reinterpret_cast<float4*>(ut)[e] =
            *reinterpret_cast<const float4*>(a.U + (b0 + j) * a.K + k0 + 4 * c4);
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            acc[r][c] = 0.0f;
#pragma unroll 4
    for (int j = 0; j < GB; ++j) {
        const float4 e0 = reinterpret_cast<const float4*>(es + j * TR)[ty];
        const float4 e1 = reinterpret_cast<const float4*>(es + j * TR + TR / 2)[ty];
        const float4 u0 = reinterpret_cast<const float4*>(ut + j * TC)[tx];
        const float er[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
        const float uc[4] = {u0.x, u0.y, u0.z, u0.w};
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[r][c] = __fmaf_rn(er[r], uc[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int64_t row = r0 + (r < 4 ? 4 * ty + r : TR / 2 + 4 * ty + r - 4);
        if (row >= a.rows)
            continue;
        float4* p = reinterpret_cast<float4*>(a.work + row * a.K + k0 + 4 * tx);
        float4 v = *p;
        v.x = __fsub_rn(v.x, acc[r][0]);
        v.y = __fsub_rn(v.y, acc[r][1]);
        v.z = __fsub_rn(v.z, acc[r][2]);
        v.w = __fsub_rn(v.w, acc[r][3]);
        *p = v;
    }
}

}  // namespace

cudaError_t launch_gptq(const GptqArgs& a, cudaStream_t st)
{
    if (a.K % GB != 0 || a.rows <= 0 || (a.rows + TR - 1) / TR > 65535 || a.rows * a.K > ((int64_t)1 << 40))
        return cudaErrorInvalidValue;
    const size_t batch_smem = sizeof(float) * GB * GB;
    const size_t trail_smem = sizeof(float) * GB * (TR + TC);
    cudaError_t e = cudaFuncSetAttribute(gptq_batch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)batch_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gptq_trailing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)trail_smem);
    if (e != cudaSuccess)
        return e;
    const int64_t n = a.rows * a.K;
    e = launch_pdl(gptq_gather_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, a);
    const unsigned row_ctas = (unsigned)((a.rows + ROWS_PER_CTA - 1) / ROWS_PER_CTA);
    const unsigned row_tiles = (unsigned)((a.rows + TR - 1) / TR);
    for (int64_t b0 = 0; b0 < a.K && e == cudaSuccess; b0 += GB) {
        e = launch_pdl(gptq_batch_kernel, dim3(row_ctas), dim3(ROWS_PER_CTA * 32), batch_smem, st, a, b0);
        const int64_t rest = a.K - b0 - GB;
        if (e == cudaSuccess && rest > 0)
            e = launch_pdl(gptq_trailing_kernel, dim3((unsigned)(rest / TC), row_tiles), dim3(TTHREADS),
                           trail_smem, st, a, b0);
    }
    return e;
}

}  // namespace fp4q
