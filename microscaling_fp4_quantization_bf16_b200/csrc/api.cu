// api.cu -- the extern "C" entry points declared in include/fp4q.h.
//
// Host side only: validate every argument, then enqueue kernels on the
// caller's stream. Nothing is allocated and nothing is synchronised.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include <atomic>

#include <cuda.h>

#include "fp4q.h"

#include "internal.h"

using namespace fp4q;

// Count of pipeline waits that ran out (see quant_tma.cuh); one word per
// device, read and cleared by fp4q_device_errors().
__device__ unsigned int g_fp4q_device_errors;

namespace {

thread_local int g_last_cuda_error = 0;

// Test hook (fp4q_debug_fail_launches): a CUDA error code that every entry
// point reports, after validating its arguments, instead of enqueuing work.
std::atomic<int> g_injected_error{0};

fp4q_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess)
        return FP4Q_OK;
    g_last_cuda_error = (int)e;
    return FP4Q_ERR_CUDA;
}

// The injected error of the test hook, or cudaSuccess.
cudaError_t injected() { return static_cast<cudaError_t>(g_injected_error.load(std::memory_order_relaxed)); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool valid_rot(int rot) { return rot == 0 || rot == 16 || rot == 32 || rot == 64 || rot == 128; }

bool valid_sub(int sub) { return sub == 2 || sub == 4 || sub == 8 || sub == 16 || sub == 32; }

// Largest tensor accepted: 2^40 elements (far above any device's memory);
// keeps every derived index and grid size inside int64 / 2^31 blocks.
constexpr int64_t kMaxElems = (int64_t)1 << 40;

// Shared checks of format, block and rotation against the shape.
fp4q_status check_format(int64_t rows, int64_t cols, int fmt, int block, int rot)
{
    if (fmt != FP4Q_FMT_NVFP4 && fmt != FP4Q_FMT_MXFP4 && fmt != FP4Q_FMT_UE5M3)
        return FP4Q_ERR_UNSUPPORTED;
    if (fmt == FP4Q_FMT_MXFP4 && block != 32)
        return FP4Q_ERR_UNSUPPORTED;
    if (fmt != FP4Q_FMT_MXFP4 && block != 4 && block != 8 && block != 16 && block != 32)
        return FP4Q_ERR_UNSUPPORTED;
    if (!valid_rot(rot))
        return FP4Q_ERR_UNSUPPORTED;
    if (rows < 0 || cols < 0)
        return FP4Q_ERR_SHAPE;
    if (cols % block != 0 || (rot > 0 && cols % rot != 0))
        return FP4Q_ERR_SHAPE;
    if (cols > 0 && rows > kMaxElems / cols)
        return FP4Q_ERR_SHAPE;
    return FP4Q_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, looked up once (no link to libcuda).
EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Which loader feeds an eligible quantize call (flattened length a multiple of
// 64, not a search; both kernels compute the same bits). By default the
// TMA-fed kernel takes MXFP4 behind a 64- or 128-wide rotation -- measured on
// B200: 66 against 78 us on a 16384 x 8192 tensor (its 4-stage copy ring hides
// the load latency that, with the cross-lane butterfly stages, bounds the
// direct kernel) -- and the direct-load kernel everything else (faster there,
// e.g. 4-over-6 behind a 16-wide rotation 107 against 111 us). FP4Q_TMA=1
// routes every eligible call to the TMA-fed kernel, FP4Q_TMA=0 none.
bool use_tma(int strat, int rot)
{
    const char* v = std::getenv("FP4Q_TMA");
    if (v != nullptr && v[0] != '\0')
        return std::strcmp(v, "0") != 0;
    return strat == K_MX && (rot == 64 || rot == 128);
}

// View of x as [n / 64, 64] bf16 rows of 128 bytes, box 64 x 64, 128-byte swizzle.
bool make_row_map(CUtensorMap* map, const void* x, int64_t n)
{
    EncodeTiledFn fn = encode_tiled();
    if (fn == nullptr)
        return false;
    cuuint64_t dims[2] = {64, (cuuint64_t)(n / 64)};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, (cuuint32_t)TMA_TILE_ROWS};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_quant(int block, int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    const bool tma_shape = a.n % 64 == 0 && a.n / 64 < ((int64_t)1 << 31);
    const bool tma_strat = strat != K_BRUTE_FORCE && strat != K_MX_BRUTE && !is_ue_strat(strat);
    if (tma_strat && tma_shape && use_tma(strat, rot)) {
        CUtensorMap map;
        if (make_row_map(&map, a.x, a.n)) {
            int dev = 0, sms = 0;
            unsigned* err = nullptr;
            cudaError_t e = cudaGetDevice(&dev);
            if (e == cudaSuccess)
                e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e == cudaSuccess)
                e = cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_fp4q_device_errors);
            if (e != cudaSuccess)
                return e;
            const int64_t ntiles = (a.n / 64 + TMA_TILE_ROWS - 1) / TMA_TILE_ROWS;
            switch (block) {
            case 4: return launch_quant_tma_b4(strat, rot, a, map, ntiles, err, sms, st);
            case 8: return launch_quant_tma_b8(strat, rot, a, map, ntiles, err, sms, st);
            case 16: return launch_quant_tma_b16(strat, rot, a, map, ntiles, err, sms, st);
            case 32: return launch_quant_tma_b32(strat, rot, a, map, ntiles, err, sms, st);
            default: return cudaErrorInvalidValue;
            }
        }
    }
    switch (block) {
    case 4: return launch_quant_b4(strat, rot, a, st);
    case 8: return launch_quant_b8(strat, rot, a, st);
    case 16: return launch_quant_b16(strat, rot, a, st);
    case 32: return launch_quant_b32(strat, rot, a, st);
    default: return cudaErrorInvalidValue;
    }
}

// NVFP4 global abs-max without a caller value: zero the output float, fold
// the tensor's abs-max into it (atomicMax on the bits), and return it as the
// amax pointer for the kernel that follows.
fp4q_status accumulate_amax(const void* x, int64_t n, int rot, float* global_scale_out,
                            cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(global_scale_out, 0, sizeof(float), st);
    if (e != cudaSuccess)
        return cuda_status(e);
    return cuda_status(launch_amax(static_cast<const uint16_t*>(x), n, rot,
                                   reinterpret_cast<unsigned*>(global_scale_out), st));
}

}  // namespace

namespace {

// fp4q_quantize and fp4q_quantize_mma: mma != 0 writes the scale bytes in the
// block-scaled MMA layout instead of row-major.
fp4q_status quantize_impl(const void* x, int64_t rows, int64_t cols, fp4q_format fmt, int block,
                          fp4q_strategy strat, int rot, const float* global_amax_in,
                          float* global_scale_out, uint8_t* codes, uint8_t* scales,
                          float* block_mse, void* dq, fp4q_dtype dq_dtype, bool mma,
                          cudaStream_t stream)
{
    fp4q_status st = check_format(rows, cols, fmt, block, rot);
    if (st != FP4Q_OK)
        return st;
    if (strat < FP4Q_ABSMAX || strat > FP4Q_BRUTE_FORCE)
        return FP4Q_ERR_UNSUPPORTED;
    if (fmt == FP4Q_FMT_MXFP4 && strat != FP4Q_ABSMAX && strat != FP4Q_BRUTE_FORCE)
        return FP4Q_ERR_UNSUPPORTED;
    if (dq != nullptr && dq_dtype != FP4Q_OUT_F32 && dq_dtype != FP4Q_OUT_BF16)
        return FP4Q_ERR_UNSUPPORTED;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t n = rows * cols;
    if (nv && global_scale_out == nullptr)
        return FP4Q_ERR_NULL;
    if (n > 0 && (x == nullptr || codes == nullptr || scales == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(block_mse) ||
        !aligned16(dq))
        return FP4Q_ERR_ALIGN;
    if (nv && (!aligned4(global_scale_out) || !aligned4(global_amax_in)))
        return FP4Q_ERR_ALIGN;
    if (nv && global_amax_in != nullptr && global_amax_in == global_scale_out)
        return FP4Q_ERR_ALIAS;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    if (n == 0)
        return nv ? cuda_status(launch_set_one(global_scale_out, stream)) : FP4Q_OK;

    QuantArgs a;
    a.x = static_cast<const uint16_t*>(x);
    a.n = n;
    a.codes = codes;
    a.scales = scales;
    a.mse = block_mse;
    a.dq = dq;
    a.dq_kind = dq == nullptr ? 0 : (dq_dtype == FP4Q_OUT_F32 ? 1 : 2);
    a.amax = nullptr;
    a.sg_out = nullptr;
    a.keep = 0xFFFFFFFFu;
    a.mma_spr = 0;
    a.mma_atoms_k = 0;
    if (mma) {  // cols % 32 == 0 and rows * cols / 32 < 2^32 (checked by the caller)
        a.mma_spr = (uint32_t)(cols / 32);
        a.mma_atoms_k = (uint32_t)((cols / block + 3) / 4);
    }
    int kstrat = nv ? (int)strat : (strat == FP4Q_BRUTE_FORCE ? K_MX_BRUTE : K_MX);
    if (fmt == FP4Q_FMT_UE5M3)
        kstrat = K_UE_ABSMAX + (int)strat;
    if (nv) {
        if (global_amax_in != nullptr) {
            a.amax = global_amax_in;
            a.sg_out = global_scale_out;
        } else {
            st = accumulate_amax(x, n, rot, global_scale_out, stream);
            if (st != FP4Q_OK)
                return st;
            a.amax = global_scale_out;  // holds the abs-max until finalised below
        }
    }
    st = cuda_status(launch_quant(block, kstrat, rot, a, stream));
    if (st != FP4Q_OK)
        return st;
    if (nv && global_amax_in == nullptr)
        st = cuda_status(launch_finalize_sg(global_scale_out, stream));
    return st;
}

}  // namespace

namespace fp4q {

fp4q_status gemm_args_status(const uint8_t* a_codes, const uint8_t* a_mma_scales,
                             const float* a_global_scale, const uint8_t* b_codes,
                             const uint8_t* b_mma_scales, const float* b_global_scale, int64_t M,
                             int64_t N, int64_t K, int fmt, const void* d, int d_dtype)
{
    if (fmt != FP4Q_FMT_NVFP4 && fmt != FP4Q_FMT_MXFP4)
        return FP4Q_ERR_UNSUPPORTED;
    if (d_dtype != FP4Q_OUT_F32 && d_dtype != FP4Q_OUT_BF16)
        return FP4Q_ERR_UNSUPPORTED;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t nalign = d_dtype == FP4Q_OUT_F32 ? 4 : 8;  // 16-byte output rows
    if (M <= 0 || N <= 0 || K <= 0 || K % 32 != 0 || N % nalign != 0 || M > 0x7FFFFFFF ||
        N > 0x7FFFFFFF || K > 0x7FFFFFFF)
        return FP4Q_ERR_SHAPE;
    if (a_codes == nullptr || a_mma_scales == nullptr || b_codes == nullptr ||
        b_mma_scales == nullptr || d == nullptr)
        return FP4Q_ERR_NULL;
    if (nv && (a_global_scale == nullptr || b_global_scale == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(a_codes) || !aligned16(a_mma_scales) || !aligned16(b_codes) ||
        !aligned16(b_mma_scales) || !aligned16(d) ||
        (nv && (!aligned4(a_global_scale) || !aligned4(b_global_scale))))
        return FP4Q_ERR_ALIGN;
    return FP4Q_OK;
}

cudaError_t injected_launch_error() { return injected(); }

fp4q_status record_cuda_error(cudaError_t e) { return cuda_status(e); }

}  // namespace fp4q

extern "C" {

fp4q_status fp4q_quantize(const void* x, int64_t rows, int64_t cols, fp4q_format fmt, int block,
                          fp4q_strategy strat, int rot, const float* global_amax_in,
                          float* global_scale_out, uint8_t* codes, uint8_t* scales,
                          float* block_mse, void* dq, fp4q_dtype dq_dtype, cudaStream_t stream)
{
    return quantize_impl(x, rows, cols, fmt, block, strat, rot, global_amax_in, global_scale_out,
                         codes, scales, block_mse, dq, dq_dtype, false, stream);
}

fp4q_status fp4q_quantize_mma(const void* x, int64_t rows, int64_t cols, fp4q_format fmt,
                              fp4q_strategy strat, int rot, const float* global_amax_in,
                              float* global_scale_out, uint8_t* codes, uint8_t* mma_scales,
                              cudaStream_t stream)
{
    if (fmt != FP4Q_FMT_NVFP4 && fmt != FP4Q_FMT_MXFP4)
        return FP4Q_ERR_UNSUPPORTED;
    if (rows < 0 || cols < 0 || cols % 32 != 0 || (rows > 0 && rows * (cols / 32) > 0xFFFFFFFFll) ||
        rows > 0x7FFFFFFF)
        return FP4Q_ERR_SHAPE;
    return quantize_impl(x, rows, cols, fmt, fmt == FP4Q_FMT_NVFP4 ? 16 : 32, strat, rot,
                         global_amax_in, global_scale_out, codes, mma_scales, nullptr, nullptr,
                         FP4Q_OUT_F32, true, stream);
}

fp4q_status fp4q_dequantize(const uint8_t* codes, const uint8_t* scales,
                            const float* global_scale, int64_t rows, int64_t cols,
                            fp4q_format fmt, int block, void* out, fp4q_dtype out_dtype,
                            cudaStream_t stream)
{
    fp4q_status st = check_format(rows, cols, fmt, block, 0);
    if (st != FP4Q_OK)
        return st;
    if (out_dtype != FP4Q_OUT_F32 && out_dtype != FP4Q_OUT_BF16)
        return FP4Q_ERR_UNSUPPORTED;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t n = rows * cols;
    if (n == 0)
        return FP4Q_OK;
    if (codes == nullptr || scales == nullptr || out == nullptr || (nv && global_scale == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(out) || (nv && !aligned4(global_scale)))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    DequantArgs a;
    a.codes = codes;
    a.scales = scales;
    a.sg = nv ? global_scale : nullptr;
    a.n = n;
    a.out = out;
    a.out_kind = out_dtype == FP4Q_OUT_F32 ? 1 : 2;
    a.keep = 0xFFFFFFFFu;
    return cuda_status(launch_dequant((int)fmt, block, a, stream));
}

fp4q_status fp4q_dequantize_unrotate(const uint8_t* codes, const uint8_t* scales,
                                     const float* global_scale, int64_t rows, int64_t cols,
                                     fp4q_format fmt, int block, int rot, void* out,
                                     fp4q_dtype out_dtype, cudaStream_t stream)
{
    fp4q_status st = check_format(rows, cols, fmt, block, rot);
    if (st != FP4Q_OK)
        return st;
    if (out_dtype != FP4Q_OUT_F32 && out_dtype != FP4Q_OUT_BF16)
        return FP4Q_ERR_UNSUPPORTED;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t n = rows * cols;
    if (n == 0)
        return FP4Q_OK;
    if (codes == nullptr || scales == nullptr || out == nullptr || (nv && global_scale == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(out) || (nv && !aligned4(global_scale)))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    DequantArgs a;
    a.codes = codes;
    a.scales = scales;
    a.sg = nv ? global_scale : nullptr;
    a.n = n;
    a.out = out;
    a.out_kind = out_dtype == FP4Q_OUT_F32 ? 1 : 2;
    a.keep = 0xFFFFFFFFu;
    return cuda_status(launch_dequant_rot((int)fmt, block, rot, a, stream));
}

size_t fp4q_mma_scale_bytes(int64_t rows, int64_t K, fp4q_format fmt)
{
    const int sfv = fmt == FP4Q_FMT_NVFP4 ? 16 : (fmt == FP4Q_FMT_MXFP4 ? 32 : 0);
    if (sfv == 0 || rows <= 0 || K <= 0 || K % sfv != 0 || rows > 0x7FFFFFFF || K > 0x7FFFFFFF)
        return 0;
    return mma_scale_bytes(rows, K, sfv);
}

fp4q_status fp4q_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t K, fp4q_format fmt,
                               uint8_t* mma_scales, cudaStream_t stream)
{
    if (fmt != FP4Q_FMT_NVFP4 && fmt != FP4Q_FMT_MXFP4)
        return FP4Q_ERR_UNSUPPORTED;
    const int sfv = fmt == FP4Q_FMT_NVFP4 ? 16 : 32;
    if (rows <= 0 || K <= 0 || K % sfv != 0 || rows > 0x7FFFFFFF || K > 0x7FFFFFFF)
        return FP4Q_ERR_SHAPE;
    if (scales == nullptr || mma_scales == nullptr)
        return FP4Q_ERR_NULL;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    return cuda_status(launch_scales_to_mma(scales, rows, K, sfv, mma_scales, stream));
}

fp4q_status fp4q_gemm(const uint8_t* a_codes, const uint8_t* a_mma_scales,
                      const float* a_global_scale, const uint8_t* b_codes,
                      const uint8_t* b_mma_scales, const float* b_global_scale, int64_t M,
                      int64_t N, int64_t K, fp4q_format fmt, float* alpha_out, void* d,
                      fp4q_dtype d_dtype, cudaStream_t stream)
{
    fp4q_status st0 = fp4q::gemm_args_status(a_codes, a_mma_scales, a_global_scale, b_codes,
                                             b_mma_scales, b_global_scale, M, N, K, fmt, d, d_dtype);
    if (st0 != FP4Q_OK)
        return st0;
    if (alpha_out == nullptr)
        return FP4Q_ERR_NULL;
    if (!aligned4(alpha_out))
        return FP4Q_ERR_ALIGN;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    fp4q_status st = cuda_status(
        launch_alpha(nv ? a_global_scale : nullptr, nv ? b_global_scale : nullptr, alpha_out, stream));
    if (st != FP4Q_OK)
        return st;
    const int m = (int)M, n = (int)N, k = (int)K;
    cudaError_t e;
    if (nv)
        e = d_dtype == FP4Q_OUT_F32
                ? launch_gemm_nv_f32(a_codes, a_mma_scales, b_codes, b_mma_scales, m, n, k, alpha_out, d, stream)
                : launch_gemm_nv_bf16(a_codes, a_mma_scales, b_codes, b_mma_scales, m, n, k, alpha_out, d, stream);
    else
        e = d_dtype == FP4Q_OUT_F32
                ? launch_gemm_mx_f32(a_codes, a_mma_scales, b_codes, b_mma_scales, m, n, k, alpha_out, d, stream)
                : launch_gemm_mx_bf16(a_codes, a_mma_scales, b_codes, b_mma_scales, m, n, k, alpha_out, d, stream);
    return cuda_status(e);
}

fp4q_status fp4q_block_mse(const void* x, const uint8_t* codes, const uint8_t* scales,
                           const float* global_scale, int64_t rows, int64_t cols,
                           fp4q_format fmt, int block, int rot, float* block_mse,
                           cudaStream_t stream)
{
    fp4q_status st = check_format(rows, cols, fmt, block, rot);
    if (st != FP4Q_OK)
        return st;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t n = rows * cols;
    if (n == 0)
        return FP4Q_OK;
    if (x == nullptr || codes == nullptr || scales == nullptr || block_mse == nullptr ||
        (nv && global_scale == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(block_mse) ||
        (nv && !aligned4(global_scale)))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    MseArgs a;
    a.x = static_cast<const uint16_t*>(x);
    a.codes = codes;
    a.scales = scales;
    a.sg = nv ? global_scale : nullptr;
    a.n = n;
    a.mse = block_mse;
    return cuda_status(launch_block_mse((int)fmt, block, rot, a, stream));
}

fp4q_status fp4q_focus_fwd(const void* w, const void* c, int64_t rows, int64_t cols,
                           fp4q_format fmt, int block, int sub, const float* global_amax_in,
                           float* global_scale_out, void* w_hat, fp4q_dtype out_dtype,
                           uint8_t* codes, uint8_t* scales, cudaStream_t stream)
{
    fp4q_status st = check_format(rows, cols, fmt, block, 0);
    if (st != FP4Q_OK)
        return st;
    if (fmt == FP4Q_FMT_UE5M3)
        return FP4Q_ERR_UNSUPPORTED;  // FOCUS is defined for MXFP4 and NVFP4
    if (!valid_sub(sub) || sub > block)
        return FP4Q_ERR_UNSUPPORTED;
    if (out_dtype != FP4Q_OUT_F32 && out_dtype != FP4Q_OUT_BF16)
        return FP4Q_ERR_UNSUPPORTED;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t n = rows * cols;
    if (nv && global_scale_out == nullptr)
        return FP4Q_ERR_NULL;
    if (n > 0 && (w == nullptr || c == nullptr || w_hat == nullptr))
        return FP4Q_ERR_NULL;
    if (n > 0 && (codes == nullptr) != (scales == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(w) || !aligned16(c) || !aligned16(w_hat) || !aligned16(codes) || !aligned16(scales))
        return FP4Q_ERR_ALIGN;
    if (nv && (!aligned4(global_scale_out) || !aligned4(global_amax_in)))
        return FP4Q_ERR_ALIGN;
    if (nv && global_amax_in != nullptr && global_amax_in == global_scale_out)
        return FP4Q_ERR_ALIAS;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    if (n == 0)
        return nv ? cuda_status(launch_set_one(global_scale_out, stream)) : FP4Q_OK;

    FocusFwdArgs a;
    a.w = static_cast<const uint16_t*>(w);
    a.c = static_cast<const uint16_t*>(c);
    a.n = n;
    a.amax = nullptr;
    a.sg_out = nullptr;
    a.w_hat = w_hat;
    a.out_kind = out_dtype == FP4Q_OUT_F32 ? 1 : 2;
    a.codes = codes;
    a.scales = scales;
    a.keep = 0xFFFFFFFFu;
    if (nv) {
        if (global_amax_in != nullptr) {
            a.amax = global_amax_in;
            a.sg_out = global_scale_out;
        } else {
            st = accumulate_amax(w, n, 0, global_scale_out, stream);
            if (st != FP4Q_OK)
                return st;
            a.amax = global_scale_out;
        }
    }
    st = cuda_status(launch_focus_fwd(nv ? 0 : 1, block, sub, a, stream));
    if (st != FP4Q_OK)
        return st;
    if (nv && global_amax_in == nullptr)
        st = cuda_status(launch_finalize_sg(global_scale_out, stream));
    return st;
}

fp4q_status fp4q_focus_bwd(const void* w, const void* g, const void* c, int64_t rows,
                           int64_t cols, int sub, float* dc, cudaStream_t stream)
{
    if (!valid_sub(sub))
        return FP4Q_ERR_UNSUPPORTED;
    if (rows < 0 || cols < 0 || cols % sub != 0 || (cols > 0 && rows > kMaxElems / cols))
        return FP4Q_ERR_SHAPE;
    const int64_t n = rows * cols;
    if (n == 0)
        return FP4Q_OK;
    if (w == nullptr || g == nullptr || c == nullptr || dc == nullptr)
        return FP4Q_ERR_NULL;
    if (!aligned16(w) || !aligned16(g) || !aligned16(c) || !aligned16(dc))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    FocusBwdArgs a;
    a.w = static_cast<const uint16_t*>(w);
    a.g = static_cast<const uint16_t*>(g);
    a.c = static_cast<const uint16_t*>(c);
    a.n = n;
    a.dc = dc;
    return cuda_status(launch_focus_bwd(sub, a, stream));
}

namespace {

// Optimizer constants on the host: 1 - b in fp32; Adam's step size for step t
// in Kingma & Ba's efficient ordering, lr * sqrt(1 - b2^t) / (1 - b1^t),
// computed in double and rounded once to fp32.
OptConsts opt_consts(fp4q_optimizer opt, float lr, float b1, float b2, float eps, int64_t t)
{
    OptConsts o;
    o.lr = lr;
    o.b1 = b1;
    o.b2 = b2;
    o.eps = eps;
    o.om1 = 1.0f - b1;
    o.om2 = 1.0f - b2;
    o.alpha = lr;
    if (opt == FP4Q_OPT_ADAM) {
        const double bc1 = 1.0 - std::pow((double)b1, (double)t);
        const double bc2 = 1.0 - std::pow((double)b2, (double)t);
        o.alpha = (float)((double)lr * std::sqrt(bc2) / bc1);
    }
    return o;
}

// Optimizer arguments; Adam's moments are required only when there is work.
fp4q_status check_opt(fp4q_optimizer opt, int64_t t, const float* m, const float* v, int64_t n)
{
    if (opt != FP4Q_OPT_SGD && opt != FP4Q_OPT_ADAM)
        return FP4Q_ERR_UNSUPPORTED;
    if (opt == FP4Q_OPT_ADAM && t < 1)
        return FP4Q_ERR_UNSUPPORTED;
    if (n > 0 && opt == FP4Q_OPT_ADAM && (m == nullptr || v == nullptr))
        return FP4Q_ERR_NULL;
    return FP4Q_OK;
}

}  // namespace

fp4q_status fp4q_focus_update(const void* w, const void* g, float* c, void* c_half, float* m,
                              float* v, int64_t rows, int64_t cols, int sub, fp4q_optimizer opt,
                              float lr, float b1, float b2, float eps, int64_t t,
                              cudaStream_t stream)
{
    if (!valid_sub(sub))
        return FP4Q_ERR_UNSUPPORTED;
    if (rows < 0 || cols < 0 || cols % sub != 0 || (cols > 0 && rows > kMaxElems / cols))
        return FP4Q_ERR_SHAPE;
    const int64_t n = rows * cols;
    fp4q_status st = check_opt(opt, t, m, v, n);
    if (st != FP4Q_OK)
        return st;
    if (n == 0)
        return FP4Q_OK;
    if (w == nullptr || g == nullptr || c == nullptr)
        return FP4Q_ERR_NULL;
    if (!aligned16(w) || !aligned16(g) || !aligned16(c) || !aligned16(c_half) || !aligned16(m) ||
        !aligned16(v))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    const bool adam = opt == FP4Q_OPT_ADAM;
    FocusUpdateArgs a;
    a.w = static_cast<const uint16_t*>(w);
    a.g = static_cast<const uint16_t*>(g);
    a.c = c;
    a.c_half = static_cast<uint16_t*>(c_half);
    a.m = adam ? m : nullptr;
    a.v = adam ? v : nullptr;
    a.n = n;
    a.o = opt_consts(opt, lr, b1, b2, eps, t);
    return cuda_status(launch_focus_update(sub, adam, a, stream));
}

fp4q_status fp4q_focus_step(const void* w, int64_t rows, int64_t cols, fp4q_format fmt, int block,
                            int sub, const float* global_amax_in, float* global_scale_out,
                            float* c, void* c_half, float* m, float* v, float* sse,
                            fp4q_optimizer opt, float lr, float b1, float b2, float eps,
                            int64_t t, cudaStream_t stream)
{
    fp4q_status st = check_format(rows, cols, fmt, block, 0);
    if (st != FP4Q_OK)
        return st;
    if (fmt == FP4Q_FMT_UE5M3)
        return FP4Q_ERR_UNSUPPORTED;  // FOCUS is defined for MXFP4 and NVFP4
    if (!valid_sub(sub) || sub > block)
        return FP4Q_ERR_UNSUPPORTED;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t n = rows * cols;
    st = check_opt(opt, t, m, v, n);
    if (st != FP4Q_OK)
        return st;
    if (nv && global_scale_out == nullptr)
        return FP4Q_ERR_NULL;
    if (n > 0 && (w == nullptr || c == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(w) || !aligned16(c) || !aligned16(c_half) || !aligned16(m) || !aligned16(v) ||
        !aligned16(sse))
        return FP4Q_ERR_ALIGN;
    if (nv && (!aligned4(global_scale_out) || !aligned4(global_amax_in)))
        return FP4Q_ERR_ALIGN;
    if (nv && global_amax_in != nullptr && global_amax_in == global_scale_out)
        return FP4Q_ERR_ALIAS;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    if (n == 0)
        return nv ? cuda_status(launch_set_one(global_scale_out, stream)) : FP4Q_OK;

    const bool adam = opt == FP4Q_OPT_ADAM;
    FocusStepArgs a;
    a.w = static_cast<const uint16_t*>(w);
    a.n = n;
    a.amax = nullptr;
    a.sg_out = nullptr;
    a.c = c;
    a.c_half = static_cast<uint16_t*>(c_half);
    a.m = adam ? m : nullptr;
    a.v = adam ? v : nullptr;
    a.sse = sse;
    a.keep = 0xFFFFFFFFu;
    a.o = opt_consts(opt, lr, b1, b2, eps, t);
    if (nv) {
        if (global_amax_in != nullptr) {
            a.amax = global_amax_in;
            a.sg_out = global_scale_out;
        } else {
            st = accumulate_amax(w, n, 0, global_scale_out, stream);
            if (st != FP4Q_OK)
                return st;
            a.amax = global_scale_out;  // holds the abs-max until finalised below
        }
    }
    st = cuda_status(launch_focus_step(nv ? 0 : 1, block, sub, adam, a, stream));
    if (st != FP4Q_OK)
        return st;
    if (nv && global_amax_in == nullptr)
        st = cuda_status(launch_finalize_sg(global_scale_out, stream));
    return st;
}

fp4q_status fp4q_gptq(const void* w, int64_t rows, int64_t cols, fp4q_format fmt, int block,
                      int rot, const uint8_t* scales, const float* global_scale, const float* U,
                      const int32_t* perm, float* work, uint8_t* codes, cudaStream_t stream)
{
    fp4q_status st = check_format(rows, cols, fmt, block, rot);
    if (st != FP4Q_OK)
        return st;
    if (cols % 128 != 0 || rows > 0x7FFFFFFF)
        return FP4Q_ERR_SHAPE;
    if (rot > 0 && cols * 4 > kGptqRowBytes)
        return FP4Q_ERR_SHAPE;
    const bool nv = fmt == FP4Q_FMT_NVFP4;
    const int64_t n = rows * cols;
    if (n == 0)
        return FP4Q_OK;
    if (w == nullptr || scales == nullptr || U == nullptr || work == nullptr || codes == nullptr ||
        (nv && global_scale == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(w) || !aligned16(scales) || !aligned16(U) || !aligned16(perm) ||
        !aligned16(work) || !aligned16(codes) || (nv && !aligned4(global_scale)))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    GptqArgs a;
    a.w = static_cast<const uint16_t*>(w);
    a.scales = scales;
    a.sg = nv ? global_scale : nullptr;
    a.U = U;
    a.perm = perm;
    a.work = work;
    a.codes = codes;
    a.rows = rows;
    a.K = cols;
    a.fmt = (int)fmt;
    a.block = block;
    a.rot = rot;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&a.err), g_fp4q_device_errors);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(codes, 0, (size_t)(n / 2), stream);
    if (e == cudaSuccess)
        e = launch_gptq(a, stream);
    return cuda_status(e);
}

fp4q_status fp4q_global_amax(const void* x, int64_t rows, int64_t cols, int rot, float* amax_out,
                             cudaStream_t stream)
{
    if (!valid_rot(rot))
        return FP4Q_ERR_UNSUPPORTED;
    if (rows < 0 || cols < 0 || (rot > 0 && cols % rot != 0) || (cols > 0 && rows > kMaxElems / cols))
        return FP4Q_ERR_SHAPE;
    const int64_t n = rows * cols;
    if (amax_out == nullptr || (n > 0 && x == nullptr))
        return FP4Q_ERR_NULL;
    if (!aligned16(x) || !aligned4(amax_out))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), stream);
    if (e != cudaSuccess || n == 0)
        return cuda_status(e);
    return cuda_status(
        launch_amax(static_cast<const uint16_t*>(x), n, rot, reinterpret_cast<unsigned*>(amax_out), stream));
}

fp4q_status fp4q_e2m1_encode(const float* u, int64_t n, uint8_t* out, cudaStream_t stream)
{
    if (n < 0 || n > kMaxElems)
        return FP4Q_ERR_SHAPE;
    if (n == 0)
        return FP4Q_OK;
    if (u == nullptr || out == nullptr)
        return FP4Q_ERR_NULL;
    if (!aligned16(u) || !aligned16(out))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    return cuda_status(launch_e2m1_encode(u, n, out, stream));
}

fp4q_status fp4q_e4m3_encode(const float* v, int64_t n, uint8_t* out, cudaStream_t stream)
{
    if (n < 0 || n > kMaxElems)
        return FP4Q_ERR_SHAPE;
    if (n == 0)
        return FP4Q_OK;
    if (v == nullptr || out == nullptr)
        return FP4Q_ERR_NULL;
    if (!aligned16(v) || !aligned16(out))
        return FP4Q_ERR_ALIGN;
    if (cudaError_t ie = injected())
        return cuda_status(ie);
    return cuda_status(launch_e4m3_encode(v, n, out, stream));
}

const char* fp4q_status_string(fp4q_status s)
{
    switch (s) {
    case FP4Q_OK: return "ok";
    case FP4Q_ERR_NULL: return "a required pointer is NULL";
    case FP4Q_ERR_SHAPE: return "invalid shape (negative, or cols not a multiple of block/rot/sub)";
    case FP4Q_ERR_ALIGN: return "pointer not aligned (16 bytes for arrays, 4 for scalars)";
    case FP4Q_ERR_UNSUPPORTED: return "unsupported format/block/strategy/rotation/sub/dtype";
    case FP4Q_ERR_ALIAS: return "global_amax_in and global_scale_out alias";
    case FP4Q_ERR_CUDA: return "CUDA launch error (see fp4q_last_cuda_error)";
    default: return "unknown status";
    }
}

int fp4q_last_cuda_error(void) { return g_last_cuda_error; }

void fp4q_debug_fail_launches(int cuda_error) { g_injected_error.store(cuda_error); }

int fp4q_device_errors(void)
{
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_fp4q_device_errors, sizeof(v)) != cudaSuccess)
        return -1;
    if (v != 0 && cudaMemcpyToSymbol(g_fp4q_device_errors, &zero, sizeof(zero)) != cudaSuccess)
        return -1;
    return (int)v;
}

}  // extern "C"
