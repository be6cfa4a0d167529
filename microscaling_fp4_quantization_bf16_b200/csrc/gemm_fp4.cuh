// gemm_fp4.cuh -- W4A4 block-scaled FP4 GEMM on the 5th-generation tensor
// cores: D[M, N] = alpha * sum_k A[m, k] B[n, k] with A (activations) and B
// (weights) as packed E2M1 codes, K contiguous, and one E4M3 (NVFP4, per 16
// elements) or E8M0 (MXFP4, per 32) scale per block, in the layout the
// block-scaled MMA reads (fp4q_scales_to_mma). This is the consumer of the
// quantizer's output ("Bridging the Gap Between Promise and Performance for
// Microscaling FP4 Quantization", 技術概要 §2.3: MXFP4 / NVFP4 matrix
// multiplication on Blackwell SM100).
//
// The kernel is CUTLASS's SM100 block-scaled collective (tcgen05.mma
// kind::mxf4nvf4 with block scales, TMA-fed shared-memory stages, TMEM
// accumulators), instantiated here with a 128x128x256 tile and a 1x1x1
// cluster: every TMA load is a plain single-CTA copy. No source matrix C is read.
#pragma once

#include <cuda_runtime.h>

#include "cute/tensor.hpp"
#include "cutlass/cutlass.h"
#include "cutlass/detail/sm100_blockscaled_layout.hpp"
#include "cutlass/epilogue/collective/collective_builder.hpp"
#include "cutlass/gemm/collective/collective_builder.hpp"
#include "cutlass/gemm/device/gemm_universal_adapter.h"
#include "cutlass/gemm/dispatch_policy.hpp"
#include "cutlass/gemm/kernel/gemm_universal.hpp"
#include "cutlass/numeric_types.h"
#include "cutlass/util/packed_stride.hpp"

// CuTe reports a tensor-map encode that the driver rejects only through
// assert() (after printing the descriptor's fields); compiled with NDEBUG the
// GEMM would then be launched with that descriptor. Keep assertions on here.
#ifdef NDEBUG
#error "the GEMM units must be compiled with assertions enabled (see above)"
#endif

// One GEMM configuration in its own namespace: ELEM_A is the CUTLASS
// block-scaled FP4 type, ELEM_D the output type.
#define FP4Q_GEMM_CONFIG(NS, ELEM_A, ELEM_D)                                                      \
    namespace NS {                                                                                \
    using namespace cute;                                                                         \
    using ElementA = ELEM_A;                                                                      \
    using ElementB = ELEM_A;                                                                      \
    using LayoutA = cutlass::layout::RowMajor;                                                    \
    using LayoutB = cutlass::layout::ColumnMajor;                                                 \
    constexpr int AlignA = 32, AlignB = 32;                                                       \
    using ElementC = void;                                                                        \
    using ElementD = ELEM_D;                                                                      \
    using LayoutC = cutlass::layout::RowMajor;                                                    \
    using LayoutD = cutlass::layout::RowMajor;                                                    \
    constexpr int AlignD = 128 / cutlass::sizeof_bits<ElementD>::value;                           \
    constexpr int AlignC = AlignD;                                                                \
    using Acc = float;                                                                            \
    using Tile = Shape<_128, _128, _256>;                                                         \
    using Cluster = Shape<_1, _1, _1>;                                                            \
    using Epi = typename cutlass::epilogue::collective::CollectiveBuilder<                        \
        cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, Tile, Cluster,                      \
        cutlass::epilogue::collective::EpilogueTileAuto, Acc, Acc, ElementC, LayoutC, AlignC,     \
        ElementD, LayoutD, AlignD, cutlass::epilogue::collective::EpilogueScheduleAuto>::CollectiveOp; \
    using Main = typename cutlass::gemm::collective::CollectiveBuilder<                           \
        cutlass::arch::Sm100, cutlass::arch::OpClassBlockScaledTensorOp, ElementA, LayoutA,       \
        AlignA, ElementB, LayoutB, AlignB, Acc, Tile, Cluster,                                    \
        cutlass::gemm::collective::StageCountAutoCarveout<static_cast<int>(                       \
            sizeof(typename Epi::SharedStorage))>,                                                \
        cutlass::gemm::collective::KernelScheduleAuto>::CollectiveOp;                             \
    using Kernel = cutlass::gemm::kernel::GemmUniversal<Shape<int, int, int, int>, Main, Epi,     \
                                                        void>;                                   \
    using Gemm = cutlass::gemm::device::GemmUniversalAdapter<Kernel>;                             \
    }

namespace fp4q {

// Runs D = alpha * A B^T for one configuration. Scale buffers are in the MMA
// layout of the same problem shape; alpha is read from device memory.
template <class Gemm>
cudaError_t run_fp4_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb,
                         int M, int N, int K, const float* alpha, void* d, cudaStream_t st)
{
    using namespace cute;
    using Kernel = typename Gemm::GemmKernel;
    using Mainloop = typename Kernel::CollectiveMainloop;
    using Config = typename Mainloop::Sm1xxBlkScaledConfig;
    using EA = typename Mainloop::ArrayElementA;
    using EB = typename Mainloop::ArrayElementB;
    using ESF = typename Mainloop::ElementSF;
    using ED = typename Kernel::CollectiveEpilogue::ElementD;
    auto lsa = Config::tile_atom_to_shape_SFA(make_shape(M, N, K, 1));
    auto lsb = Config::tile_atom_to_shape_SFB(make_shape(M, N, K, 1));
    auto sA = cutlass::make_cute_packed_stride(typename Kernel::StrideA{}, {M, K, 1});
    auto sB = cutlass::make_cute_packed_stride(typename Kernel::StrideB{}, {N, K, 1});
    auto sC = cutlass::make_cute_packed_stride(typename Kernel::StrideC{}, {M, N, 1});
    auto sD = cutlass::make_cute_packed_stride(typename Kernel::StrideD{}, {M, N, 1});
    typename Gemm::Arguments args{
        cutlass::gemm::GemmUniversalMode::kGemm,
        {M, N, K, 1},
        {reinterpret_cast<EA const*>(a), sA, reinterpret_cast<EB const*>(b), sB,
         reinterpret_cast<ESF const*>(sfa), lsa, reinterpret_cast<ESF const*>(sfb), lsb},
        {{}, nullptr, sC, reinterpret_cast<ED*>(d), sD}};
    args.epilogue.thread.alpha = 1.0f;
    args.epilogue.thread.beta = 0.0f;
    args.epilogue.thread.alpha_ptr = alpha;
    // The driver rejects every tensor-map encode once the context holds an
    // error (a kernel that faulted earlier leaves a sticky one, 700 for an
    // illegal address): report it here instead of reaching the encode.
    if (cudaError_t e = cudaPeekAtLastError(); e != cudaSuccess)
        return e;
    Gemm g;
    if (g.can_implement(args) != cutlass::Status::kSuccess)
        return cudaErrorInvalidValue;
    if (Gemm::get_workspace_size(args) != 0)  // the library allocates nothing
        return cudaErrorInvalidValue;
    if (g.initialize(args, nullptr, st) != cutlass::Status::kSuccess)
        return cudaErrorInvalidValue;
    if (g.run(st) != cutlass::Status::kSuccess) {
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? cudaErrorLaunchFailure : e;
    }
    return cudaGetLastError();
}

}  // namespace fp4q
