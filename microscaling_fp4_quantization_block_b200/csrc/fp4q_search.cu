// fp4q_search.cu -- dispatch of the MSE-optimised scale search kernels
// ("Bridging the Gap", s3, MR-GPTQ: MSE-optimised grids) for every scale
// format, block size and rotation.
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

template <int FMT, int B, int K>
cudaError_t run_search(const QuantParams& p, cudaStream_t s)
{
    auto kern = search_kernel<FMT, B, K>;
    const int grid = grid_for((const void*)kern, ring_smem_bytes<K>(), ring_ctas_needed(p.n, EPT));
    return launch_pdl(kern, grid, kThreads, ring_smem_bytes<K>(), s, p);
}

template <int FMT, int B>
cudaError_t search_by_rot(int K, const QuantParams& p, cudaStream_t s)
{
    switch (K) {
    case 0: return run_search<FMT, B, 0>(p, s);
    case 16: return run_search<FMT, B, 16>(p, s);
    case 32: return run_search<FMT, B, 32>(p, s);
    case 128: return run_search<FMT, B, 128>(p, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t search_by_block(int B, int K, const QuantParams& p, cudaStream_t s)
{
    switch (B) {
    case 8: return search_by_rot<FMT, 8>(K, p, s);
    case 16: return search_by_rot<FMT, 16>(K, p, s);
    case 32: return search_by_rot<FMT, 32>(K, p, s);
    case 64: return search_by_rot<FMT, 64>(K, p, s);
    case 128: return search_by_rot<FMT, 128>(K, p, s);
    case 256: return search_by_rot<FMT, 256>(K, p, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_quantize_search(int fmt, int B, int K, const QuantParams& p, cudaStream_t s)
{
    switch (fmt) {
    case kE8M0: return search_by_block<kE8M0>(B, K, p, s);
    case kUE4M3: return search_by_block<kUE4M3>(B, K, p, s);
    case kUE5M3: return search_by_block<kUE5M3>(B, K, p, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace fp4q
