// fp4q_quantize_ue5m3.cu -- quantize kernels with ue5m3 block scales.
#include "fp4q_quantize_impl.cuh"

namespace fp4q {

cudaError_t launch_quantize_ue5m3(int B, int K, bool mse, const QuantParams& p, int* grid_out, cudaStream_t s)
{
    return detail::by_block<kUE5M3>(B, K, mse, p, grid_out, s);
}

}  // namespace fp4q
