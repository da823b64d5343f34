// fp4q_dequantize.cu -- template dispatch of the dequantize and block-MSE kernels.
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

template <int B, int K, bool F32>
cudaError_t run_dequantize(const DequantParams& p, cudaStream_t s)
{
    if constexpr (K <= kDqChunk) {
        // rotation runs of at most 16: interleaved chunks, fully coalesced stores
        auto kern = dequantize_il_kernel<B, K, F32>;
        const int64_t tiles = (p.n + kDqTile - 1) / kDqTile;
        const int grid = grid_for((const void*)kern, kRingBytesPerCta, (tiles + kWarps - 1) / kWarps);
        return launch_pdl(kern, grid, kThreads, kRingBytesPerCta, s, p);
    } else {
        auto kern = dequantize_kernel<B, K, F32>;
        const int64_t tile_elems = 32 * DPL;  // 32 lanes x 128 elements
        const int64_t tiles = (p.n + tile_elems - 1) / tile_elems;
        const int grid = grid_for((const void*)kern, kRingBytesPerCta, (tiles + kWarps - 1) / kWarps);
        return launch_pdl(kern, grid, kThreads, kRingBytesPerCta, s, p);
    }
}

template <int B, int K>
cudaError_t deq_out(bool f32, const DequantParams& p, cudaStream_t s)
{
    return f32 ? run_dequantize<B, K, true>(p, s) : run_dequantize<B, K, false>(p, s);
}

template <int B, int K>
cudaError_t run_mse(const MseParams& p, int* grid_out, cudaStream_t s)
{
    auto kern = block_mse_kernel<B, K>;
    int64_t need = ring_ctas_needed(p.n, EPT);
    if (need > partial_slots(p.n)) need = partial_slots(p.n);
    const int grid = grid_for((const void*)kern, ring_smem_bytes<K>(), need);
    *grid_out = grid;
    return launch_pdl(kern, grid, kThreads, ring_smem_bytes<K>(), s, p);
}

#define FP4Q_BK_SWITCH(B, K, CALL)                                                   \
    switch (B) {                                                                     \
    case 8: FP4Q_K_SWITCH(8, K, CALL)                                                \
    case 16: FP4Q_K_SWITCH(16, K, CALL)                                              \
    case 32: FP4Q_K_SWITCH(32, K, CALL)                                              \
    case 64: FP4Q_K_SWITCH(64, K, CALL)                                              \
    case 128: FP4Q_K_SWITCH(128, K, CALL)                                            \
    case 256: FP4Q_K_SWITCH(256, K, CALL)                                            \
    default: break;                                                                  \
    }
#define FP4Q_K_SWITCH(BB, K, CALL)                                                   \
    switch (K) {                                                                     \
    case 0: CALL(BB, 0)                                                              \
    case 16: CALL(BB, 16)                                                            \
    case 32: CALL(BB, 32)                                                            \
    case 128: CALL(BB, 128)                                                          \
    default: break;                                                                  \
    }                                                                                \
    break;

}  // namespace

cudaError_t launch_dequantize(int B, int K, bool f32out, const DequantParams& p, cudaStream_t s)
{
#define DEQ_CALL(BB, KK) return deq_out<BB, KK>(f32out, p, s);
    FP4Q_BK_SWITCH(B, K, DEQ_CALL)
#undef DEQ_CALL
    return cudaErrorInvalidValue;
}

cudaError_t launch_block_mse(int B, int K, const MseParams& p, int* grid_out, cudaStream_t s)
{
#define MSE_CALL(BB, KK) return run_mse<BB, KK>(p, grid_out, s);
    FP4Q_BK_SWITCH(B, K, MSE_CALL)
#undef MSE_CALL
    return cudaErrorInvalidValue;
}

}  // namespace fp4q
