// fp4q_quantize_e8m0.cu -- quantize kernels with e8m0 block scales.
#include "fp4q_quantize_impl.cuh"

namespace fp4q {

cudaError_t launch_quantize_e8m0(int B, int K, bool mse, const QuantParams& p, int* grid_out, cudaStream_t s)
{
    return detail::by_block<kE8M0>(B, K, mse, p, grid_out, s);
}

// MXFP4 (block 32) only: the batched fused quantizer of a model's weight pass.
cudaError_t launch_quantize_batch_e8m0(int B, int K, const QuantBatchParams& p, cudaStream_t s)
{
    if (B != 32) return cudaErrorInvalidValue;
    return detail::batch_by_rot<kE8M0, 32>(K, p, s);
}

}  // namespace fp4q
