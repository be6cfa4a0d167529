// gemm_noalloc.cu -- fp4q_gemm_noalloc: fp4q_gemm with the library's own
// scratch float for alpha instead of a caller-owned one.
//
// fp4q_gemm writes alpha = s_g(A) * s_g(B) into a device float before the GEMM
// kernel reads it, and asks the caller for that float. Some callers cannot
// supply one on the call path: a serving loop whose memory comes from a pool
// sized once at start-up, or code that must not call the allocator between
// launches (an allocation can synchronise the device or fail under memory
// pressure, and neither may happen while a batch is in flight). For them this
// entry point uses a small array that lives in the library image itself.
#include <cuda_runtime.h>

#include <mutex>

#include "fp4q.h"
#include "internal.h"

namespace {

// Scratch floats of this entry point: alpha needs one. The array has a fixed
// size of 256 bytes, and the use is checked against it at compile time (no
// call can ask for more).
constexpr int kScratchFloats = 64;
constexpr int kAlphaFloats = 1;
static_assert(kAlphaFloats <= kScratchFloats, "scratch too small for alpha");

static __device__ __align__(256) float g_gemm_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_addr_lock;
float* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up with
// cudaGetSymbolAddress on the first call per device and cached for the life
// of the process. The cache is not invalidated: after cudaDeviceReset the
// module is loaded again (possibly at another address), so a process that
// resets a device must not call this entry point on it afterwards.
cudaError_t scratch_address(float** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_addr_lock);
    if (g_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gemm_scratch);
        if (e != cudaSuccess)
            return e;
        g_addr[dev] = static_cast<float*>(p);
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" fp4q_status fp4q_gemm_noalloc(const uint8_t* a_codes, const uint8_t* a_mma_scales,
                                         const float* a_global_scale, const uint8_t* b_codes,
                                         const uint8_t* b_mma_scales,
                                         const float* b_global_scale, int64_t M, int64_t N,
                                         int64_t K, fp4q_format fmt, void* d, fp4q_dtype d_dtype,
                                         cudaStream_t stream)
{
    fp4q_status st = fp4q::gemm_args_status(a_codes, a_mma_scales, a_global_scale, b_codes,
                                            b_mma_scales, b_global_scale, M, N, K, fmt, d, d_dtype);
    if (st != FP4Q_OK)
        return st;
    if (cudaError_t ie = fp4q::injected_launch_error())
        return fp4q::record_cuda_error(ie);
    float* alpha = nullptr;
    if (cudaError_t e = scratch_address(&alpha))
        return fp4q::record_cuda_error(e);
    // alpha is written by the first kernel of the call before the GEMM reads it;
    // nothing in the scratch has to start at zero.
    return fp4q_gemm(a_codes, a_mma_scales, a_global_scale, b_codes, b_mma_scales, b_global_scale,
                     M, N, K, fmt, alpha, d, d_dtype, stream);
}
