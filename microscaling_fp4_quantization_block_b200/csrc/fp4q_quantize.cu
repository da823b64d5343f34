// fp4q_quantize.cu -- template dispatch of the quantize and amax kernels.
#include <mutex>
#include <unordered_map>

#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {

int resident_grid(const void* kernel, int64_t ctas_needed)
{
    static std::mutex mu;
    static std::unordered_map<uint64_t, int> cache;   // (kernel, device) -> resident CTAs
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t key = reinterpret_cast<uint64_t>(kernel) * 64u + (uint64_t)dev;
    int resident = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) resident = it->second;
    }
    if (resident == 0) {
        int sms = 0, occ = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, 0);
        resident = (sms > 0 ? sms : 1) * (occ > 0 ? occ : 1);
        std::lock_guard<std::mutex> lock(mu);
        cache[key] = resident;
    }
    if (ctas_needed < 1) ctas_needed = 1;
    return (int)(ctas_needed < resident ? ctas_needed : resident);
}

namespace {

template <int FMT, int B, int K>
cudaError_t run_quantize(const QuantParams& p, cudaStream_t s)
{
    auto kern = quantize_kernel<FMT, B, K>;
    const int64_t tiles = (p.n + kTileElems - 1) / kTileElems;
    const int grid = resident_grid((const void*)kern, (tiles + kThreads / 32 - 1) / (kThreads / 32));
    kern<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <int FMT, int B>
cudaError_t by_rot(int K, const QuantParams& p, cudaStream_t s)
{
    switch (K) {
    case 0: return run_quantize<FMT, B, 0>(p, s);
    case 16: return run_quantize<FMT, B, 16>(p, s);
    case 32: return run_quantize<FMT, B, 32>(p, s);
    case 128: return run_quantize<FMT, B, 128>(p, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t by_block(int B, int K, const QuantParams& p, cudaStream_t s)
{
    switch (B) {
    case 8: return by_rot<FMT, 8>(K, p, s);
    case 16: return by_rot<FMT, 16>(K, p, s);
    case 32: return by_rot<FMT, 32>(K, p, s);
    case 64: return by_rot<FMT, 64>(K, p, s);
    case 128: return by_rot<FMT, 128>(K, p, s);
    case 256: return by_rot<FMT, 256>(K, p, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int K>
cudaError_t run_amax(const AmaxParams& p, cudaStream_t s)
{
    auto kern = amax_kernel<K>;
    const int64_t tiles = (p.n + kTileElems - 1) / kTileElems;
    const int grid = resident_grid((const void*)kern, (tiles + kThreads / 32 - 1) / (kThreads / 32));
    kern<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(int fmt, int B, int K, const QuantParams& p, cudaStream_t s)
{
    switch (fmt) {
    case kE8M0: return by_block<kE8M0>(B, K, p, s);
    case kUE4M3: return by_block<kUE4M3>(B, K, p, s);
    case kUE5M3: return by_block<kUE5M3>(B, K, p, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_amax(int K, const AmaxParams& p, cudaStream_t s)
{
    switch (K) {
    case 0: return run_amax<0>(p, s);
    case 16: return run_amax<16>(p, s);
    case 32: return run_amax<32>(p, s);
    case 128: return run_amax<128>(p, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace fp4q
