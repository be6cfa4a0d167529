// quant_b8.cu -- instantiations of the quantize kernel for block size 8.
#include "quant_kernel.cuh"

namespace fp4q {
cudaError_t launch_quant_b8(int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    return launch_quant_impl<8>(strat, rot, a, st);
}
}  // namespace fp4q
