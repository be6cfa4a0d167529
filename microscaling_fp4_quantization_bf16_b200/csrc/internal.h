// internal.h -- argument blocks and launcher declarations shared between the
// C-ABI layer (api.cu) and the kernel translation units.
#pragma once

#include <cstdint>
#include <utility>

#include <cuda.h>
#include <cuda_runtime_api.h>

#include "fp4q.h"

namespace fp4q {

// Host-side helpers of the C-ABI layer (api.cu). gemm_args_status: the
// argument checks of fp4q_gemm other than alpha_out. injected_launch_error:
// the error set with fp4q_debug_fail_launches, or cudaSuccess.
// record_cuda_error: FP4Q_ERR_CUDA with e kept for fp4q_last_cuda_error (or
// FP4Q_OK for cudaSuccess).
fp4q_status gemm_args_status(const uint8_t* a_codes, const uint8_t* a_mma_scales,
                             const float* a_global_scale, const uint8_t* b_codes,
                             const uint8_t* b_mma_scales, const float* b_global_scale, int64_t M,
                             int64_t N, int64_t K, int fmt, const void* d, int d_dtype);
cudaError_t injected_launch_error();
fp4q_status record_cuda_error(cudaError_t e);

// Launch with programmatic stream serialization (see pdl_begin in
// fp4q_device.cuh); returns the launch status.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Strategy ids used by the kernels (NVFP4 strategies follow the ABI enum;
// MXFP4 abs-max is its own kernel family).
enum KStrat { K_ABSMAX = 0, K_PREVENT_ZERO = 1, K_FOUR_OVER_SIX = 2, K_BRUTE_FORCE = 3, K_MX = 4,
              K_MX_BRUTE = 5,
              // UE5M3 block scales (no global scale), the four strategies in order
              K_UE_ABSMAX = 6, K_UE_PREVENT_ZERO = 7, K_UE_FOUR_OVER_SIX = 8, K_UE_BRUTE_FORCE = 9 };

__host__ __device__ constexpr bool is_ue_strat(int s) { return s >= K_UE_ABSMAX && s <= K_UE_BRUTE_FORCE; }
__host__ __device__ constexpr bool is_mx_strat(int s) { return s == K_MX || s == K_MX_BRUTE; }

struct QuantArgs {
    const uint16_t* x;      // bf16 [n]
    int64_t n;              // elements (rows * cols)
    const float* amax;      // NVFP4: device tensor abs-max; NULL for MXFP4
    float* sg_out;          // NVFP4: receives s_g from thread 0 of block 0, or NULL
    uint8_t* codes;         // [n / 2]
    uint8_t* scales;        // [n / B]
    float* mse;             // [n / B] or NULL
    void* dq;               // [n] or NULL
    int dq_kind;            // 0 none, 1 fp32, 2 bf16
    uint32_t keep;          // 0xFFFFFFFF, passed at run time (see encode_seg)
    uint32_t mma_spr;       // 0: row-major scales; else segments per row, and scales are
                            // written in the block-scaled MMA layout (see gemm_sf.cu)
    uint32_t mma_atoms_k;   // MMA layout: 4-block atoms per 128-row tile along K
};

struct DequantArgs {
    const uint8_t* codes;
    const uint8_t* scales;
    const float* sg;        // NVFP4 global scale (device), NULL for MXFP4
    int64_t n;
    void* out;
    int out_kind;           // 1 fp32, 2 bf16
    uint32_t keep;          // 0xFFFFFFFF, passed at run time (see dequant_rot_kernel)
};

struct MseArgs {
    const uint16_t* x;
    const uint8_t* codes;
    const uint8_t* scales;
    const float* sg;
    int64_t n;
    float* mse;
};

struct FocusFwdArgs {
    const uint16_t* w;      // bf16 [n]
    const uint16_t* c;      // fp16 [n / sub]
    int64_t n;
    const float* amax;      // NVFP4 tensor abs-max (device)
    float* sg_out;
    void* w_hat;
    int out_kind;           // 1 fp32, 2 bf16
    uint8_t* codes;         // optional
    uint8_t* scales;        // optional
    uint32_t keep;          // 0xFFFFFFFF, passed at run time (see encode_seg)
};

struct FocusBwdArgs {
    const uint16_t* w;
    const uint16_t* g;
    const uint16_t* c;
    int64_t n;
    float* dc;
};

// Optimizer constants of one FOCUS calibration step; om1 = 1 - b1 and
// om2 = 1 - b2 in fp32; alpha = Adam's step size for this step (lr for SGD).
struct OptConsts {
    float lr, b1, b2, om1, om2, alpha, eps;
};

struct FocusUpdateArgs {
    const uint16_t* w;      // bf16 [n]
    const uint16_t* g;      // bf16 [n]
    float* c;               // fp32 [n / sub], in place
    uint16_t* c_half;       // fp16 [n / sub], optional
    float* m;               // Adam moments [n / sub] (Adam only)
    float* v;
    int64_t n;
    OptConsts o;
};

struct FocusStepArgs {
    const uint16_t* w;      // bf16 [n]
    int64_t n;
    const float* amax;      // NVFP4 tensor abs-max (device)
    float* sg_out;
    float* c;
    uint16_t* c_half;
    float* m;
    float* v;
    float* sse;             // fp32 [n / sub], optional
    uint32_t keep;          // 0xFFFFFFFF, passed at run time (see encode_seg)
    OptConsts o;
};

// GPTQ error feedback with static groups (gptq.cu).
struct GptqArgs {
    const uint16_t* w;      // bf16 [rows, K], original column order
    const uint8_t* scales;  // [rows, K / block] fixed block scales
    const float* sg;        // NVFP4 s_g (device), else unused
    const float* U;         // fp32 [K, K] upper Cholesky factor of H^-1, processing order
    const int32_t* perm;    // [K] processing position -> column, or NULL
    float* work;            // fp32 [rows, K] scratch
    uint8_t* codes;         // [rows, K / 2], zeroed by the caller
    unsigned* err;          // device error counter
    int64_t rows, K;
    int fmt, block;         // fmt: 0 NVFP4, 1 MXFP4, 2 UE5M3
    int rot;                // 0, or the width of the blockwise rotation applied first
};

// Largest row (bytes of fp32) the rotated GPTQ path stages in shared memory.
constexpr int64_t kGptqRowBytes = 227 * 1024;

// Each launcher returns cudaErrorInvalidValue for a combination it does not
// provide (the ABI layer validates before calling), else the launch status.
cudaError_t launch_quant_b4(int strat, int rot, const QuantArgs& a, cudaStream_t st);
cudaError_t launch_quant_b8(int strat, int rot, const QuantArgs& a, cudaStream_t st);
cudaError_t launch_quant_b16(int strat, int rot, const QuantArgs& a, cudaStream_t st);
cudaError_t launch_quant_b32(int strat, int rot, const QuantArgs& a, cudaStream_t st);

// TMA-fed quantize kernel (flattened length a multiple of 64; not brute force).
// The tensor map views x as [n / 64, 64] bf16 with 128-byte swizzle and a box
// of 64 x 64; ntiles = ceil(n / 64 / 64); err is the device error word.
constexpr int TMA_TILE_ROWS = 64;
cudaError_t launch_quant_tma_b4(int strat, int rot, const QuantArgs& a, const CUtensorMap& map,
                                int64_t ntiles, unsigned* err, int sms, cudaStream_t st);
cudaError_t launch_quant_tma_b8(int strat, int rot, const QuantArgs& a, const CUtensorMap& map,
                                int64_t ntiles, unsigned* err, int sms, cudaStream_t st);
cudaError_t launch_quant_tma_b16(int strat, int rot, const QuantArgs& a, const CUtensorMap& map,
                                 int64_t ntiles, unsigned* err, int sms, cudaStream_t st);
cudaError_t launch_quant_tma_b32(int strat, int rot, const QuantArgs& a, const CUtensorMap& map,
                                 int64_t ntiles, unsigned* err, int sms, cudaStream_t st);

cudaError_t launch_amax(const uint16_t* x, int64_t n, int rot, unsigned* out, cudaStream_t st);
cudaError_t launch_finalize_sg(float* g, cudaStream_t st);
cudaError_t launch_set_one(float* p, cudaStream_t st);
// fmt: 0 NVFP4, 1 MXFP4, 2 UE5M3 (the fp4q_format values).
cudaError_t launch_dequant(int fmt, int block, const DequantArgs& a, cudaStream_t st);
cudaError_t launch_dequant_rot(int fmt, int block, int rot, const DequantArgs& a, cudaStream_t st);
cudaError_t launch_block_mse(int fmt, int block, int rot, const MseArgs& a, cudaStream_t st);
cudaError_t launch_focus_fwd(int mx, int block, int sub, const FocusFwdArgs& a, cudaStream_t st);
cudaError_t launch_focus_bwd(int sub, const FocusBwdArgs& a, cudaStream_t st);
cudaError_t launch_focus_update(int sub, bool adam, const FocusUpdateArgs& a, cudaStream_t st);
cudaError_t launch_gptq(const GptqArgs& a, cudaStream_t st);
cudaError_t launch_focus_step(int mx, int block, int sub, bool adam, const FocusStepArgs& a,
                              cudaStream_t st);
// W4A4 FP4 GEMM (gemm_*.cu): scale layout for the block-scaled MMA and the
// four GEMM configurations (NVFP4 / MXFP4 x fp32 / bf16 output).
size_t mma_scale_bytes(int64_t rows, int64_t K, int sfv);
cudaError_t launch_scales_to_mma(const uint8_t* src, int64_t rows, int64_t K, int sfv, uint8_t* dst,
                                 cudaStream_t st);
cudaError_t launch_alpha(const float* sga, const float* sgb, float* alpha, cudaStream_t st);
#define FP4Q_DECLARE_GEMM(NAME)                                                                  \
    cudaError_t NAME(const uint8_t* a, const uint8_t* sfa, const uint8_t* b, const uint8_t* sfb, \
                     int M, int N, int K, const float* alpha, void* d, cudaStream_t st);
FP4Q_DECLARE_GEMM(launch_gemm_nv_f32)
FP4Q_DECLARE_GEMM(launch_gemm_nv_bf16)
FP4Q_DECLARE_GEMM(launch_gemm_mx_f32)
FP4Q_DECLARE_GEMM(launch_gemm_mx_bf16)
#undef FP4Q_DECLARE_GEMM
cudaError_t launch_e2m1_encode(const float* u, int64_t n, uint8_t* out, cudaStream_t st);
cudaError_t launch_e4m3_encode(const float* v, int64_t n, uint8_t* out, cudaStream_t st);

}  // namespace fp4q
