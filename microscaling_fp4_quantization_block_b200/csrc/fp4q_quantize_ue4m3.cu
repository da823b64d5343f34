// fp4q_quantize_ue4m3.cu -- quantize kernels with ue4m3 block scales.
#include "fp4q_quantize_impl.cuh"

namespace fp4q {

cudaError_t launch_quantize_ue4m3(int B, int K, bool mse, const QuantParams& p, int* grid_out, cudaStream_t s)
{
    return detail::by_block<kUE4M3>(B, K, mse, p, grid_out, s);
}

// NVFP4 (block 16) only: the batched fused quantizer of a model's weight pass.
cudaError_t launch_quantize_batch_ue4m3(int B, int K, const QuantBatchParams& p, cudaStream_t s)
{
    if (B != 16) return cudaErrorInvalidValue;
    return detail::batch_by_rot<kUE4M3, 16>(K, p, s);
}

}  // namespace fp4q
