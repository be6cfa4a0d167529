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
//   gptq_rotate_gather_kernel  work[i][j] = W[i][perm[j]] widened to fp32, the
//                        row staged in shared memory (rotated blockwise first
//                        when MR-GPTQ's rotation is asked for, as the
//                        quantizer rotates it); gptq_gather_kernel for rows
//                        too long to stage
//   gptq_batch_kernel    first applies the previous batch's update to its
//                        own 128 columns (the trailing arithmetic below),
//                        then eight rows per warp (four lanes each) run the
//                        batch's 128 positions in order: quantize with the
//                        fixed scale, error e = (w - value * S) / U[j][j],
//                        spread inside the batch (w_k = fma(-e, U[j][k], w_k));
//                        the codes go to their original column, e replaces
//                        the dead weight in work
//   gptq_trailing_kernel the columns from two batches on: t = fma chain of
//                        e_j * U[j][k] over the batch (j ascending, from 0),
//                        w_k -= t; a persistent fp32 CUDA-core GEMM without
//                        split-K, so each element's sum has the fixed order.
//                        It runs concurrently with the next batch kernel
//                        (launch_gptq gives the stream order), which is the
//                        sequential part of the method.
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
constexpr int QL = 4;             // batch kernel: lanes per row
constexpr int QR = 32 / QL;       // rows per warp
constexpr int QC = GB / (4 * QL); // chunks of 4 consecutive positions per lane
constexpr int QWARPS = 4;         // warps per CTA
constexpr int Q_ROWS = QR * QWARPS;
constexpr int TR = 128;           // trailing kernel: TR rows x TC columns per work item
constexpr int TC = 64;
constexpr int TX = TC / 4;        // threads across the columns
constexpr int TTHREADS = TX * (TR / 8);  // 8 rows x 4 columns of outputs per thread

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

// Dequantization scale of the scale byte b (NVFP4: times s_g, passed as sg).
__device__ __forceinline__ float scale_of(const GptqArgs& a, uint32_t b, float sg)
{
    if (a.fmt == 1)
        return e8m0_dec(b);
    if (a.fmt == 2)
        return ue5m3_dec(b);
    return __fmul_rn(e4m3_dec(b), sg);
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
// order: work[i][j] = rotated(W)[i][perm[j]]. With ROT = 0 it is the plain
// gather with the row staged in shared memory, so that the permuted reads
// hit shared memory and the row is read from HBM with 128-bit loads.
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

__device__ __forceinline__ void cp_async16(float* smem, const float* gmem)
{
    const unsigned d = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

constexpr int QWS = GB + 16;  // row stride of the staged weights: conflict-free 128-bit reads
constexpr size_t kBatchSmem = sizeof(float) * ((size_t)GB * GB + (size_t)Q_ROWS * QWS);
// The batch kernel shares an SM with a trailing-update CTA (256 threads of at
// most 176 registers): 4 warps of at most 160 registers fill the register file.
constexpr int kBatchRegs = 160;

// The previous batch's update of this batch's columns, for the CTA's Q_ROWS
// rows: t = fma chain of e_j * U[b0 - GB + j][b0 + c] over j ascending from
// 0, then w - t (the trailing kernel's arithmetic, for the columns it leaves
// out). On entry us holds that U tile (already landed); on return us holds
// U's diagonal block of this batch and stage[r][QWS] the updated weights.
// Thread (tx, ty) = (tid % 32, tid / 32): rows 8 ty .. 8 ty + 7, columns
// 4 tx .. 4 tx + 3.
__device__ __forceinline__ void fold_previous_batch(const GptqArgs& a, int64_t b0, float* us, float* stage)
{
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int64_t r0 = (int64_t)blockIdx.x * Q_ROWS;
    float* es = stage;  // [GB][Q_ROWS]: es[j][r] = error of row r0 + r at position b0 - GB + j
#pragma unroll 8
    for (int e = threadIdx.x; e < Q_ROWS * GB / 4; e += QWARPS * 32) {
        const int r = e % Q_ROWS, j4 = e / Q_ROWS;
        const int64_t row = r0 + r;
        float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (row < a.rows)
            v = __ldcg(reinterpret_cast<const float4*>(a.work + row * a.K + b0 - GB + 4 * j4));
        es[(4 * j4) * Q_ROWS + r] = v.x;
        es[(4 * j4 + 1) * Q_ROWS + r] = v.y;
        es[(4 * j4 + 2) * Q_ROWS + r] = v.z;
        es[(4 * j4 + 3) * Q_ROWS + r] = v.w;
    }
    float4 old[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int64_t row = r0 + 8 * ty + k;
        old[k] = row < a.rows ? __ldcg(reinterpret_cast<const float4*>(a.work + row * a.K + b0 + 4 * tx))
                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    __syncthreads();
    f32x2 acc[4][4];  // {local row 2p, 2p + 1} at column c
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            acc[p][c] = pk2(0.0f, 0.0f);
#pragma unroll 4
    for (int j = 0; j < GB; ++j) {
        const float4 e0 = reinterpret_cast<const float4*>(es + j * Q_ROWS + 8 * ty)[0];
        const float4 e1 = reinterpret_cast<const float4*>(es + j * Q_ROWS + 8 * ty)[1];
        const float4 u = reinterpret_cast<const float4*>(us + j * GB)[tx];
        const f32x2 ep[4] = {pk2(e0.x, e0.y), pk2(e0.z, e0.w), pk2(e1.x, e1.y), pk2(e1.z, e1.w)};
        const f32x2 ud[4] = {pk2(u.x, u.x), pk2(u.y, u.y), pk2(u.z, u.z), pk2(u.w, u.w)};
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[p][c] = fma2(ep[p], ud[c], acc[p][c]);
    }
    __syncthreads();  // the fold tile and the error tile are no longer read
    for (int e = threadIdx.x; e < GB * GB / 4; e += QWARPS * 32) {
        const int r = e / (GB / 4), c4 = e - r * (GB / 4);
        cp_async16(us + 4 * e, a.U + (b0 + r) * a.K + b0 + 4 * c4);
    }
    cp_async_commit();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        float t[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float lo, hi;
            upk2(acc[k / 2][c], lo, hi);
            t[c] = (k & 1) ? hi : lo;
        }
        const float4 o = old[k];
        *reinterpret_cast<float4*>(stage + (8 * ty + k) * QWS + 4 * tx) =
            make_float4(__fsub_rn(o.x, t[0]), __fsub_rn(o.y, t[1]), __fsub_rn(o.z, t[2]), __fsub_rn(o.w, t[3]));
    }
    cp_async_wait<0>();
    __syncthreads();
}

// QWARPS warps of QR = 8 rows (QL = 4 lanes per row) per CTA. After the
// previous batch's update of the CTA's rows (fold_previous_batch; batch 0
// reads its weights directly), lane s of a row holds the positions
// 16 c + 4 s + e (chunk c = 0..7, e = 0..3) as packed pairs, and U's
// 128 x 128 diagonal block sits in shared memory.
//
// Every lane of a row carries the weight wn of the current position (updated
// through the previous error) with its scale and reciprocal, and forms the
// error itself, so no shuffle sits between one error and the next: the next
// position's weight, short of this step's update, is fetched from its owner
// while the error is formed, and the one missing fma (the owner's operands)
// is applied after it. Each step then updates every chunk from the current
// one on with one 128-bit shared load of U's row and two packed fmas; the
// positions of those chunks already quantized take the same fma harmlessly
// (their weights are dead). Every live weight thus receives exactly the fma
// chain of the definition, in position order. The errors (which replace the
// batch's dead weights in work) and the codes are written at the end.
__global__ void __maxnreg__(kBatchRegs) gptq_batch_kernel(GptqArgs a, int64_t b0)
{
    extern __shared__ float us[];        // [GB][GB]: U's fold tile, then its diagonal block
    float* stage = us + GB * GB;         // the fold's error tile, then the batch's weights
    // U, the scales and perm are inputs of the call that no kernel of it
    // writes, so they are read before waiting for the previous kernel.
    const int64_t ur = b0 > 0 ? b0 - GB : b0;  // rows of U: the previous batch's (fold) or this one's
    for (int e = threadIdx.x; e < GB * GB / 4; e += blockDim.x) {
        const int r = e / (GB / 4), c4 = e - r * (GB / 4);
        cp_async16(us + 4 * e, a.U + (ur + r) * a.K + b0 + 4 * c4);
    }
    cp_async_commit();
    // the batch's original columns, checked once per CTA
    __shared__ int32_t pcol[GB];
    for (int j = threadIdx.x; j < GB; j += blockDim.x) {
        int32_t c = (int32_t)(b0 + j);
        if (a.perm != nullptr) {
            c = a.perm[b0 + j];
            if (c < 0 || c >= a.K) {
                atomicAdd(a.err, 1u);  // not a permutation of 0..K-1: recorded, column 0 used
                c = 0;
            }
        }
        pcol[j] = c;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int s = lane % QL;
    const int64_t i = (int64_t)blockIdx.x * Q_ROWS + (threadIdx.x >> 5) * QR + lane / QL;
    const bool live = i < a.rows;  // dead lanes still take part in the shuffles
    // independent loads of the 32 scale bytes, then their values
    const uint8_t* srow = a.scales + (live ? i : 0) * (a.K / a.block);
    const float sg = a.fmt == 0 ? *a.sg : 1.0f;
    uint32_t sb[QC][4];
#pragma unroll
    for (int c = 0; c < QC; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            sb[c][e] = srow[pcol[16 * c + 4 * s + e] / a.block];
    float S[QC][4], R[QC][4];
#pragma unroll
    for (int c = 0; c < QC; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            S[c][e] = live ? scale_of(a, sb[c][e], sg) : 0.0f;
            R[c][e] = S[c][e] == 0.0f ? 0.0f : guarded_rcp(S[c][e]);
        }
    cp_async_wait<0>();
    __syncthreads();
    pdl_begin();
    // work is read through L2 (ld.global.cg): kernels of this call run
    // concurrently (see launch_gptq), so no L1 copy of it is trusted.
    float* wr = a.work + (live ? i : 0) * a.K + b0;
    f32x2 w2[QC][2];  // {e = 0, 1}, {e = 2, 3} of chunk c
    if (b0 == 0) {
#pragma unroll
        for (int c = 0; c < QC; ++c) {
            float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (live)
                v = __ldcg(reinterpret_cast<const float4*>(wr + 16 * c + 4 * s));
            w2[c][0] = pk2(v.x, v.y);
            w2[c][1] = pk2(v.z, v.w);
        }
    } else {
        fold_previous_batch(a, b0, us, stage);
        const float* wrow = stage + (threadIdx.x / QL) * QWS;
#pragma unroll
        for (int c = 0; c < QC; ++c) {
            const float4 v = *reinterpret_cast<const float4*>(wrow + 16 * c + 4 * s);
            w2[c][0] = pk2(v.x, v.y);
            w2[c][1] = pk2(v.z, v.w);
        }
    }
    auto wval = [&](int c, int e) {
        float lo, hi;
        upk2(w2[c][e >> 1], lo, hi);
        return (e & 1) ? hi : lo;
    };
    // A position's scale is last read when its weight is fetched ahead, one
    // step before it is quantized; S[c][e] then keeps the owner's error.
    uint32_t qw[QC / 2];  // chunk c's codes at bits 16 (c % 2) + 4 e of word c / 2
#pragma unroll
    for (int k = 0; k < QC / 2; ++k)
        qw[k] = 0u;
    float wn = __shfl_sync(0xFFFFFFFFu, wval(0, 0), 0, QL);
    float Sn = __shfl_sync(0xFFFFFFFFu, S[0][0], 0, QL);
    float Rn = __shfl_sync(0xFFFFFFFFu, R[0][0], 0, QL);
#pragma unroll
    for (int c = 0; c < QC; ++c) {
        const int cn = c + 1 < QC ? c + 1 : c;
#pragma unroll 1
        for (int so = 0; so < QL; ++so) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int jj = 16 * c + 4 * so + e;
                // the next position: element e + 1 of the same lane, else
                // element 0 of the next lane (of the next chunk after lane QL - 1)
                float wx, Sx, Rx;
                if (e < 3) {
                    wx = __shfl_sync(0xFFFFFFFFu, wval(c, e + 1), so, QL);
                    Sx = __shfl_sync(0xFFFFFFFFu, S[c][e + 1], so, QL);
                    Rx = __shfl_sync(0xFFFFFFFFu, R[c][e + 1], so, QL);
                } else {
                    const bool wrap = so + 1 == QL;
                    const int src = wrap ? 0 : so + 1;
                    wx = __shfl_sync(0xFFFFFFFFu, wrap ? wval(cn, 0) : wval(c, 0), src, QL);
                    Sx = __shfl_sync(0xFFFFFFFFu, wrap ? S[cn][0] : S[c][0], src, QL);
                    Rx = __shfl_sync(0xFFFFFFFFu, wrap ? R[cn][0] : R[c][0], src, QL);
                }
                const float* urow = us + jj * GB;
                const float unext = urow[jj + 1 < GB ? jj + 1 : jj];
                const bool nz = Sn != 0.0f;
                const uint32_t q = nz ? e2m1_code1(__fmul_rn(wn, Rn)) : 0u;
                const float deq = nz ? __fmul_rn(e2m1_value1(q), Sn) : 0.0f;
                const float err = __fdiv_rn(__fsub_rn(wn, deq), urow[jj]);
                if (s == so) {
                    S[c][e] = err;
                    qw[c / 2] |= q << (16 * (c % 2) + 4 * e);
                }
                wn = __fmaf_rn(-err, unext, wx);
                Sn = Sx;
                Rn = Rx;
                const f32x2 ne = pk2(-err, -err);
#pragma unroll
                for (int c2 = c; c2 < QC; ++c2) {
                    const float4 u = *reinterpret_cast<const float4*>(urow + 16 * c2 + 4 * s);
                    w2[c2][0] = fma2(ne, pk2(u.x, u.y), w2[c2][0]);
                    w2[c2][1] = fma2(ne, pk2(u.z, u.w), w2[c2][1]);
                }
            }
        }
    }
    if (!live)
        return;
#pragma unroll
    for (int c = 0; c < QC; ++c) {
        *reinterpret_cast<float4*>(wr + 16 * c + 4 * s) = make_float4(S[c][0], S[c][1], S[c][2], S[c][3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t q = (qw[c / 2] >> (16 * (c % 2) + 4 * e)) & 0xFu;
            if (q != 0) {
                const int64_t x = i * a.K + pcol[16 * c + 4 * s + e];
                atomicOr(reinterpret_cast<unsigned*>(a.codes) + (x >> 3), q << (4u * (uint32_t)(x & 7)));
            }
        }
    }
}

// work[i][k] -= sum over the batch of e[i][j] * U[b0 + j][k] for k >= b0 + GB,
// each sum an fma chain in j order from 0. Persistent: every CTA takes a
// contiguous run of (row tile, column tile) items, row tile major, so the
// 128 x 128 error tile is loaded once per row tile; the 128 x 64 U tiles
// stream through two shared buffers by asynchronous copies, the next one in
// flight while the current one is used. Each thread accumulates 8 x 4
// outputs (rows 4ty..4ty+3 and 64+4ty.., columns 4tx..4tx+3) from three
// 128-bit shared loads per j; its old weights are fetched before the sums so
// their latency hides behind them.
__global__ void __launch_bounds__(TTHREADS, 1) gptq_trailing_kernel(GptqArgs a, int64_t b0, int64_t items,
                                                                   int64_t col_tiles)
{
    extern __shared__ float sm[];
    float* es = sm;              // [GB][TR]: es[j][r] = e of row r0 + r at position j
    float* ub = sm + GB * TR;    // 2 x [GB][TC]: ut[j][c] = U[b0 + j][k0 + c]
    // Runs concurrently with the batch kernel launched just before it (see
    // launch_gptq): it lets the next kernel launch, works, and waits for that
    // batch kernel only at its end, so its completion implies the batch's.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t first = (int64_t)blockIdx.x * items / gridDim.x;
    const int64_t last = ((int64_t)blockIdx.x + 1) * items / gridDim.x;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    auto load_u = [&](int64_t item, int buf) {
        const int64_t k0 = b0 + 2 * GB + (item % col_tiles) * TC;
        float* ut = ub + buf * (GB * TC);
        for (int e = threadIdx.x; e < GB * TC / 4; e += TTHREADS) {
            const int jj = e / (TC / 4), c4 = e - jj * (TC / 4);
            cp_async16(ut + 4 * e, a.U + (b0 + jj) * a.K + k0 + 4 * c4);
        }
        cp_async_commit();
    };
    if (first < last)
        load_u(first, 0);
    int64_t cur_rt = -1;
    int buf = 0;
    for (int64_t it = first; it < last; ++it) {
        const int64_t rt = it / col_tiles;
        const int64_t r0 = rt * TR;
        const int64_t k0 = b0 + 2 * GB + (it % col_tiles) * TC;
        if (it + 1 < last) {
            load_u(it + 1, buf ^ 1);
            cp_async_wait<1>();  // this item's U tile has landed (the next may be in flight)
        } else {
            cp_async_wait<0>();
        }
        if (rt != cur_rt) {
            __syncthreads();  // nobody still reads the previous error tile
#pragma unroll 8
            for (int e = threadIdx.x; e < TR * GB / 4; e += TTHREADS) {
                const int r = e % TR, j4 = e / TR;
                const int64_t row = r0 + r;
                float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (row < a.rows)
                    v = __ldcg(reinterpret_cast<const float4*>(a.work + row * a.K + b0 + 4 * j4));
                es[(4 * j4) * TR + r] = v.x;
                es[(4 * j4 + 1) * TR + r] = v.y;
                es[(4 * j4 + 2) * TR + r] = v.z;
                es[(4 * j4 + 3) * TR + r] = v.w;
            }
            cur_rt = rt;
        }
        __syncthreads();  // error tile and this U tile visible to all
        const float* ut = ub + buf * (GB * TC);
        float4 old[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int64_t row = r0 + (r < 4 ? 4 * ty + r : TR / 2 + 4 * ty + r - 4);
            old[r] = row < a.rows ? __ldcg(reinterpret_cast<const float4*>(a.work + row * a.K + k0 + 4 * tx))
                                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        // acc[p][c] = {sum of row 2p, sum of row 2p + 1} at column c: each lane
        // of the packed fma is the same single-rounding fma as the scalar chain
        f32x2 acc[4][4];
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[p][c] = pk2(0.0f, 0.0f);
        // PD sets of operands in flight: those of position jj + PD are loaded
        // while jj's fmas run (the last PD loads wrap to position 0: harmless).
        // Measured on the 4096 x 4096 layer: PD = 1, 2, 4 within 1%, PD = 1
        // keeps the kernel at the register count that lets a batch CTA share
        // the SM.
        constexpr int PD = 1;
        constexpr int kUnroll = 2;
        float4 pe0[PD], pe1[PD], pu0[PD];
#pragma unroll
        for (int d = 0; d < PD; ++d) {
            pe0[d] = reinterpret_cast<const float4*>(es + d * TR)[ty];
            pe1[d] = reinterpret_cast<const float4*>(es + d * TR + TR / 2)[ty];
            pu0[d] = reinterpret_cast<const float4*>(ut + d * TC)[tx];
        }
#pragma unroll kUnroll
        for (int j0 = 0; j0 < GB; j0 += PD) {
#pragma unroll
            for (int d = 0; d < PD; ++d) {
                const float4 e0 = pe0[d], e1 = pe1[d], u0 = pu0[d];
                const int jn = (j0 + d + PD) & (GB - 1);
                pe0[d] = reinterpret_cast<const float4*>(es + jn * TR)[ty];
                pe1[d] = reinterpret_cast<const float4*>(es + jn * TR + TR / 2)[ty];
                pu0[d] = reinterpret_cast<const float4*>(ut + jn * TC)[tx];
                const f32x2 ep[4] = {pk2(e0.x, e0.y), pk2(e0.z, e0.w), pk2(e1.x, e1.y), pk2(e1.z, e1.w)};
                const f32x2 ud[4] = {pk2(u0.x, u0.x), pk2(u0.y, u0.y), pk2(u0.z, u0.z), pk2(u0.w, u0.w)};
#pragma unroll
                for (int p = 0; p < 4; ++p)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        acc[p][c] = fma2(ep[p], ud[c], acc[p][c]);
            }
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
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace

cudaError_t launch_gptq(const GptqArgs& a, cudaStream_t st)
{
    if (a.K % GB != 0 || a.rows <= 0 || a.rows * a.K > ((int64_t)1 << 40))
        return cudaErrorInvalidValue;
    const size_t batch_smem = kBatchSmem;
    const size_t trail_smem = sizeof(float) * GB * (TR + 2 * TC);
    cudaError_t e = cudaFuncSetAttribute(gptq_batch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)batch_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gptq_trailing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)trail_smem);
    // A batch CTA and a trailing CTA share an SM (see the stream order below):
    // both ask for the whole shared-memory carveout, so that either finds room.
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gptq_batch_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gptq_trailing_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const int64_t n = a.rows * a.K;
    const size_t row_smem = sizeof(float) * (size_t)a.K;
    if (a.rot == 0 && (int64_t)row_smem > kGptqRowBytes) {
        // a row too long to stage: each element read through the permutation
        e = launch_pdl(gptq_gather_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, a);
    } else {
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
        case 0: e = launch_rot(gptq_rotate_gather_kernel<0>); break;
        case 16: e = launch_rot(gptq_rotate_gather_kernel<16>); break;
        case 32: e = launch_rot(gptq_rotate_gather_kernel<32>); break;
        case 64: e = launch_rot(gptq_rotate_gather_kernel<64>); break;
        case 128: e = launch_rot(gptq_rotate_gather_kernel<128>); break;
        default: e = cudaErrorInvalidValue;
        }
    }
    const unsigned row_ctas = (unsigned)((a.rows + Q_ROWS - 1) / Q_ROWS);
    const unsigned row_tiles = (unsigned)((a.rows + TR - 1) / TR);
    // Stream order: batch 0, batch 1, trailing 0, batch 2, trailing 1, ...
    // Batch b + 1 updates its own columns with batch b's errors first; the
    // trailing update of batch b covers the columns from batch b + 2 on and
    // runs concurrently with batch b + 1 (disjoint writes), ending with a wait
    // for it. Batch b + 2 waits for trailing b, hence for batch b + 1 too, and
    // each weight receives the batches' updates in batch order.
    for (int64_t b0 = 0; b0 < a.K && e == cudaSuccess; b0 += GB) {
        e = launch_pdl(gptq_batch_kernel, dim3(row_ctas), dim3(QWARPS * 32), batch_smem, st, a, b0);
        const int64_t pb = b0 - GB;  // the previous batch
        const int64_t rest = a.K - pb - 2 * GB;
        if (e == cudaSuccess && pb >= 0 && rest > 0) {
            const int64_t col_tiles = rest / TC, items = col_tiles * row_tiles;
            const unsigned ctas = (unsigned)(items < sms ? items : sms);  // one per SM
            e = launch_pdl(gptq_trailing_kernel, dim3(ctas), dim3(TTHREADS), trail_smem, st, a, pb, items,
                           col_tiles);
        }
    }
    return e;
}

}  // namespace fp4q
