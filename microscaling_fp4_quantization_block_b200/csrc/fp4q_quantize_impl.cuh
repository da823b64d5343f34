// fp4q_quantize_impl.cuh -- template dispatch of the quantize kernel for one
// scale format (each format is its own translation unit, built in parallel).
#pragma once

#include <cstring>

#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace detail {

template <int FMT, int B, int K, bool MSE, bool DQ = false>
cudaError_t run_quantize(const QuantParams& p, int* grid_out, cudaStream_t s)
{
    auto kern = quantize_kernel<FMT, B, K, MSE, DQ>;
    int64_t need = ring_ctas_needed(p.n, EPT);
    if (MSE && need > partial_slots(p.n)) need = partial_slots(p.n);
    const int grid = grid_for((const void*)kern, ring_smem_bytes<K>(), need);
    if (grid_out) *grid_out = grid;
    return launch_pdl(kern, grid, kThreads, ring_smem_bytes<K>(), s, p);
}

template <int FMT, int B, int K>
cudaError_t by_mse(bool mse, const QuantParams& p, int* g, cudaStream_t s)
{
    if (!mse) return run_quantize<FMT, B, K, false>(p, g, s);
    return p.y ? run_quantize<FMT, B, K, true, true>(p, g, s) : run_quantize<FMT, B, K, true>(p, g, s);
}

template <int FMT, int B>
cudaError_t by_rot(int K, bool mse, const QuantParams& p, int* g, cudaStream_t s)
{
    switch (K) {
    case 0: return by_mse<FMT, B, 0>(mse, p, g, s);
    case 16: return by_mse<FMT, B, 16>(mse, p, g, s);
    case 32: return by_mse<FMT, B, 32>(mse, p, g, s);
    case 128: return by_mse<FMT, B, 128>(mse, p, g, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t by_block(int B, int K, bool mse, const QuantParams& p, int* g, cudaStream_t s)
{
    switch (B) {
    case 8: return by_rot<FMT, 8>(K, mse, p, g, s);
    case 16: return by_rot<FMT, 16>(K, mse, p, g, s);
    case 32: return by_rot<FMT, 32>(K, mse, p, g, s);
    case 64: return by_rot<FMT, 64>(K, mse, p, g, s);
    case 128: return by_rot<FMT, 128>(K, mse, p, g, s);
    case 256: return by_rot<FMT, 256>(K, mse, p, g, s);
    default: return cudaErrorInvalidValue;
    }
}

// The batched fused quantizer: grid = the resident CTAs the tiles can use, at
// most kMaxPartialCtas (every tensor's workspace holds that many partials).
template <int FMT, int B, int K>
cudaError_t run_quantize_batch(const QuantBatchParams& p, cudaStream_t s)
{
    auto kern = quantize_batch_kernel<FMT, B, K>;
    int64_t need = ((int64_t)p.tile0[p.count] + kWarps - 1) / kWarps;
    if (need > kMaxPartialCtas) need = kMaxPartialCtas;
    const int grid = grid_for((const void*)kern, ring_smem_bytes<K>(), need);
    return launch_pdl(kern, grid, kThreads, ring_smem_bytes<K>(), s, p);
}

template <int FMT, int B>
cudaError_t batch_by_rot(int K, const QuantBatchParams& p, cudaStream_t s)
{
    switch (K) {
    case 0: return run_quantize_batch<FMT, B, 0>(p, s);
    case 16: return run_quantize_batch<FMT, B, 16>(p, s);
    case 32: return run_quantize_batch<FMT, B, 32>(p, s);
    case 128: return run_quantize_batch<FMT, B, 128>(p, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace detail
}  // namespace fp4q
