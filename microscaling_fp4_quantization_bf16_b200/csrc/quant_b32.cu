// quant_b32.cu -- instantiations of the quantize kernels for block size 32.
#include "quant_tma.cuh"

namespace fp4q {
cudaError_t launch_quant_b32(int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    return launch_quant_impl<32>(strat, rot, a, st);
}

cudaError_t launch_quant_tma_b32(int strat, int rot, const QuantArgs& a, const CUtensorMap& map,
                                 int64_t ntiles, unsigned* err, int sms, cudaStream_t st)
{
    return launch_quant_tma_impl<32>(strat, rot, a, map, ntiles, err, sms, st);
}
}  // namespace fp4q
