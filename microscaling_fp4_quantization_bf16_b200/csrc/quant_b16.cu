// quant_b16.cu -- instantiations of the quantize kernels for block size 16.
#include "quant_tma.cuh"

namespace fp4q {
cudaError_t launch_quant_b16(int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    return launch_quant_impl<16>(strat, rot, a, st);
}

cudaError_t launch_quant_tma_b16(int strat, int rot, const QuantArgs& a, const CUtensorMap& map,
                                 int64_t ntiles, unsigned* err, int sms, cudaStream_t st)
{
    return launch_quant_tma_impl<16>(strat, rot, a, map, ntiles, err, sms, st);
}
}  // namespace fp4q
