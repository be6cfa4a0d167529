// quant_b4.cu -- instantiations of the quantize kernel for block size 4.
#include "quant_kernel.cuh"

namespace fp4q {
cudaError_t launch_quant_b4(int strat, int rot, const QuantArgs& a, cudaStream_t st)
{
    return launch_quant_impl<4>(strat, rot, a, st);
}
}  // namespace fp4q
