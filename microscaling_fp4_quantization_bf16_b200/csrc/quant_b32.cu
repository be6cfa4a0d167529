// quant_b32.cu -- instantiations of the quantize kernel for block size 32.
#include "quant_kernel.cuh"

namespace fp4q {
cudaError_t launch_quant_b32(int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    return launch_quant_impl<32>(strat, rot, a, st);
}
}  // namespace fp4q
