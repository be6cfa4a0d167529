// gemm_sf.cu -- block scales from the quantizer's row-major layout
// ([rows, K / SFV], one byte per block of SFV elements) to the layout the
// block-scaled MMA reads: 128-row x 4-block atoms of 512 bytes (row r of the
// atom at byte 16 (r % 32) + 4 (r / 32), block j at + j), atoms ordered along
// K first, rows padded to 128 and blocks to 4 with zero bytes.
#include "cute/tensor.hpp"
#include "cutlass/detail/sm100_blockscaled_layout.hpp"
#include "fp4q_device.cuh"
#include "internal.h"

namespace fp4q {

namespace {

template <int SFV>
auto sf_layout(int64_t rows, int64_t K)
{
    using Config = cutlass::detail::Sm1xxBlockScaledConfig<SFV>;
    return Config::tile_atom_to_shape_SFA(cute::make_shape((int)rows, 1, (int)K, 1));
}

template <int SFV, class Layout>
__global__ void __launch_bounds__(256) scales_to_mma_kernel(const uint8_t* src, int64_t rows,
                                                            int64_t K, uint8_t* dst, Layout layout,
                                                            int64_t kb_pad, int64_t total)
{
    pdl_begin();
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= total)
        return;
    const int64_t r = i / kb_pad, kb = i % kb_pad;
    const int64_t nkb = K / SFV;
    const int64_t off = layout((int)r, (int)(kb * SFV), 0);
    dst[off] = (r < rows && kb < nkb) ? src[r * nkb + kb] : (uint8_t)0;
}

template <int SFV>
cudaError_t scales_to_mma_impl(const uint8_t* src, int64_t rows, int64_t K, uint8_t* dst,
                               cudaStream_t st)
{
    const auto layout = sf_layout<SFV>(rows, K);
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    const int64_t kb_pad = (K / SFV + 3) / 4 * 4;
    const int64_t total = rows_pad * kb_pad;
    const int64_t grid = (total + 255) / 256;
    if (grid <= 0 || grid > 0x7FFFFFFF)
        return cudaErrorInvalidValue;
    return launch_pdl(scales_to_mma_kernel<SFV, decltype(layout)>, dim3((unsigned)grid), dim3(256),
                      0, st, src, rows, K, dst, layout, kb_pad, total);
}

}  // namespace

size_t mma_scale_bytes(int64_t rows, int64_t K, int sfv)
{
    if (sfv == 16)
        return (size_t)cute::size(cute::filter_zeros(sf_layout<16>(rows, K)));
    return (size_t)cute::size(cute::filter_zeros(sf_layout<32>(rows, K)));
}

cudaError_t launch_scales_to_mma(const uint8_t* src, int64_t rows, int64_t K, int sfv, uint8_t* dst,
                                 cudaStream_t st)
{
    return sfv == 16 ? scales_to_mma_impl<16>(src, rows, K, dst, st)
                     : scales_to_mma_impl<32>(src, rows, K, dst, st);
}

}  // namespace fp4q
