// quant_tma.cuh -- warp-specialised, TMA-fed quantize kernel for sm_100a.
//
// The flattened bf16 tensor is viewed as rows of 64 elements (128 B). Each
// CTA is a small pipeline: one producer thread streams tiles of TILE_ROWS
// rows into a ring of STAGES shared-memory buffers with
// cp.async.bulk.tensor (TMA, single-CTA copies), completion tracked by mbarriers;
// four consumer warps take one 32-element segment per thread per tile, read
// it with four conflict-free 128-bit shared loads (the tensor map's 128-byte
// swizzle puts the 16-byte chunk c of row r at c ^ (r mod 8)), release the
// buffer, and run the same per-segment arithmetic as the direct-load kernel.
// CTAs are persistent: tile t goes to CTA t mod gridDim.x.
//
// Every mbarrier wait is bounded. A wait that runs out increments the
// device error word (read with fp4q_device_errors) and the thread leaves;
// the producer first waits, again bounded, for its own copies in flight.
#pragma once

#include <cuda.h>

#include "quant_kernel.cuh"

namespace fp4q {

constexpr int TMA_ROW_ELEMS = 64;                        // one 128-byte row
constexpr int TILE_ROWS = TMA_TILE_ROWS;                 // 8 KB per stage
constexpr int TILE_BYTES = TILE_ROWS * TMA_ROW_ELEMS * 2;
constexpr int TILE_SEGS = TILE_ROWS * TMA_ROW_ELEMS / SEG;  // 128 segments
#ifndef FP4Q_TMA_STAGES
#define FP4Q_TMA_STAGES 4
#endif
#ifndef FP4Q_TMA_MINB
#define FP4Q_TMA_MINB 1
#endif
constexpr int STAGES = FP4Q_TMA_STAGES;
constexpr int CONSUMER_WARPS = TILE_SEGS / 32;           // one segment per thread
constexpr int TTHREADS = (CONSUMER_WARPS + 1) * 32;      // + one producer warp
constexpr uint32_t WAIT_LIMIT = 1u << 24;                // polls before giving up
constexpr size_t TMA_SMEM_BYTES = STAGES * TILE_BYTES + 2 * STAGES * sizeof(uint64_t) + 1024;

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Waits for the phase of parity `parity` to complete; false after WAIT_LIMIT polls.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    for (uint32_t i = 0; i < WAIT_LIMIT; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done)
            return true;
    }
    return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

template <int B, int ROT, int STRAT>
__global__ void __launch_bounds__(TTHREADS, FP4Q_TMA_MINB)
    quant_tma_kernel(const __grid_constant__ CUtensorMap tmap, QuantArgs a, int64_t ntiles,
                     unsigned* err)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * TILE_BYTES);
    uint64_t* empty = full + STAGES;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x & 31;

    pdl_begin();
    __shared__ ScaleTables<STRAT> tab;
    build_scale_tables<STRAT>(tab, a);
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(full + s), 1);
            mbar_init(smem_addr(empty + s), CONSUMER_WARPS);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == CONSUMER_WARPS) {  // producer
        if (lane != 0)
            return;
        int it = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int stage = it % STAGES;
            if (it >= STAGES && !mbar_wait(smem_addr(empty + stage), ((it / STAGES) & 1) ^ 1)) {
                atomicAdd(err, 1u);
                // wait for the copies this thread still has in flight
                for (int j = it - STAGES; j < it; ++j)
                    if (j >= 0)
                        (void)mbar_wait(smem_addr(full + (j % STAGES)), (j / STAGES) & 1);
                return;
            }
            mbar_arrive_expect_tx(smem_addr(full + stage), TILE_BYTES);
            tma_load_2d(smem_addr(smem + stage * TILE_BYTES), &tmap, 0, (int)(tile * TILE_ROWS),
                        smem_addr(full + stage));
        }
        return;
    }

    // consumers: thread c takes segment c of every tile (row c/2, half c%2)
    const int c = threadIdx.x;
    const int row = c >> 1;
    const int half = c & 1;
    const int64_t nseg = a.n / SEG;
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int stage = it % STAGES;
        const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(smem_addr(full + stage), (it / STAGES) & 1));
        if (!ok) {
            if (lane == 0)
                atomicAdd(err, 1u);
            return;
        }
        const uint8_t* rowp = smem + stage * TILE_BYTES + row * 128;
        uint4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[k] = *reinterpret_cast<const uint4*>(rowp + 16 * ((half * 4 + k) ^ (row & 7)));
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_addr(empty + stage));

        float y[SEG];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            y[8 * k + 0] = bf_lo(v[k].x);
            y[8 * k + 1] = bf_hi(v[k].x);
            y[8 * k + 2] = bf_lo(v[k].y);
            y[8 * k + 3] = bf_hi(v[k].y);
            y[8 * k + 4] = bf_lo(v[k].z);
            y[8 * k + 5] = bf_hi(v[k].z);
            y[8 * k + 6] = bf_lo(v[k].w);
            y[8 * k + 7] = bf_hi(v[k].w);
        }
        // 64/128-wide chunks: neighbouring lanes of this warp
        rotate_seg<ROT, !foldable<ROT, STRAT>()>(y, lane);
        const int64_t s = tile * TILE_SEGS + c;
        if (s < nseg)  // rows past the end were zero-filled by TMA
            process_segment<B, STRAT, ROT>(y, s, SEG, a, tab);
    }
}

// Launch of the TMA kernel for one (block, strategy, rotation).
template <int B, int ROT, int STRAT>
cudaError_t launch_tma_one(const CUtensorMap& map, const QuantArgs& a, int64_t ntiles,
                           unsigned* err, int sms, cudaStream_t st)
{
    auto kern = quant_tma_kernel<B, ROT, STRAT>;
    int per_sm = 0;
    cudaError_t e = cudaSuccess;
    if (TMA_SMEM_BYTES > 48 * 1024)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TMA_SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, TTHREADS, TMA_SMEM_BYTES);
    if (e != cudaSuccess)
        return e;
    per_sm = per_sm < 1 ? 1 : per_sm;
    const int64_t grid = ntiles < (int64_t)sms * per_sm ? ntiles : (int64_t)sms * per_sm;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(TTHREADS), TMA_SMEM_BYTES, st, map, a, ntiles,
                      err);
}

template <int B>
cudaError_t launch_quant_tma_impl(int strat, int rot, const QuantArgs& a, const CUtensorMap& map,
                                  int64_t ntiles, unsigned* err, int sms, cudaStream_t st)
{
#define FP4Q_TCASE(S_, R_)                                                   \
    if (strat == S_ && rot == R_)                                            \
        return launch_tma_one<B, R_, S_>(map, a, ntiles, err, sms, st);
#define FP4Q_TROTS(S_) \
    FP4Q_TCASE(S_, 0)  \
    FP4Q_TCASE(S_, 16) \
    FP4Q_TCASE(S_, 32) \
    FP4Q_TCASE(S_, 64) \
    FP4Q_TCASE(S_, 128)
    FP4Q_TROTS(K_ABSMAX)
    FP4Q_TROTS(K_PREVENT_ZERO)
    FP4Q_TROTS(K_FOUR_OVER_SIX)
    if constexpr (B == 32) {
        FP4Q_TROTS(K_MX)
    }
#undef FP4Q_TROTS
#undef FP4Q_TCASE
    return cudaErrorInvalidValue;
}

}  // namespace fp4q
