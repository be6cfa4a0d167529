// W4A4 NVFP4 GEMM, bf16 output (see gemm_fp4.cuh).
#include "gemm_fp4.cuh"
#include "internal.h"

FP4Q_GEMM_CONFIG(fp4q_gemm_nv_bf16, cutlass::nv_float4_t<cutlass::float_e2m1_t>, cutlass::bfloat16_t)

namespace fp4q {

cudaError_t launch_gemm_nv_bf16(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                              const uint8_t* sfb, int M, int N, int K, const float* alpha, void* d,
                              cudaStream_t st)
{
    return run_fp4_gemm<fp4q_gemm_nv_bf16::Gemm>(a, sfa, b, sfb, M, N, K, alpha, d, st);
}

}  // namespace fp4q
