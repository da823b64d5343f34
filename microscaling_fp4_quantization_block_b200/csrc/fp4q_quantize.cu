// fp4q_quantize.cu -- launch helpers, format dispatch of quantize, and the amax kernels.
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {

// 0 at load; a tensor-core kernel whose bounded wait on an MMA gives up sets it to 1.
static __device__ unsigned int g_device_fault;

unsigned int* device_fault_word()
{
    static std::mutex mu;
    static std::unordered_map<int, unsigned int*> addr;   // device -> address of g_device_fault
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = addr.find(dev);
    if (it != addr.end()) return it->second;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_fault) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
    return static_cast<unsigned int*>(p);
}

int resident_ctas(const void* kernel, int smem, int threads)
{
    static std::mutex mu;
    static std::unordered_map<uint64_t, int> cache;   // (kernel, device) -> resident CTAs
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t key = (reinterpret_cast<uint64_t>(kernel) * 64u + (uint64_t)dev) * 4096u + (uint64_t)threads;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    if (smem > 48 * 1024) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    // Prefer the largest shared-memory carveout: these kernels stage their input in
    // shared memory and barely use L1, and without a preference the carveout may be
    // sized for a single CTA, capping residency at one CTA per SM.
    cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    int sms = 0, occ = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem);
    // The same bound from the kernel's registers, shared memory and threads (the
    // occupancy query reports one CTA per SM for kernels that use tensor memory;
    // the hardware co-schedules more, up to these limits).
    cudaFuncAttributes fa;
    int smem_sm = 0, smem_rsv = 0, thr_sm = 0;
    if (cudaFuncGetAttributes(&fa, kernel) == cudaSuccess &&
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) == cudaSuccess) {
        const int warps = (threads + 31) / 32;
        const int regs_warp = ((fa.numRegs * 32 + 255) / 256) * 256;
        const int by_regs = regs_warp > 0 ? 65536 / (regs_warp * warps) : 32;
        const int cta_smem = (int)fa.sharedSizeBytes + smem + smem_rsv;
        const int by_smem = cta_smem > 0 ? smem_sm / cta_smem : 32;
        const int by_thr = thr_sm / (warps * 32);
        int manual = by_regs < by_smem ? by_regs : by_smem;
        if (by_thr < manual) manual = by_thr;
        if (manual > 32) manual = 32;
        if (manual > occ) occ = manual;
    }
    const int resident = (sms > 0 ? sms : 1) * (occ > 0 ? occ : 1);
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = resident;
    return resident;
}

int grid_for(const void* kernel, int smem, int64_t ctas_needed, int threads)
{
    const int resident = resident_ctas(kernel, smem, threads);
    if (ctas_needed < 1) ctas_needed = 1;
    return (int)(ctas_needed < resident ? ctas_needed : resident);
}

int64_t ring_ctas_needed(int64_t n, int ept)
{
    (void)ept;                                   // a tile is 32 lanes x 32 elements for every unit size
    const int64_t tiles = (n + 1023) / 1024;
    return (tiles + kWarps - 1) / kWarps;
}

cudaError_t launch_quantize(int fmt, int B, int K, bool mse, const QuantParams& p, int* grid_out,
                            cudaStream_t s)
{
    switch (fmt) {
    case kE8M0: return launch_quantize_e8m0(B, K, mse, p, grid_out, s);
    case kUE4M3: return launch_quantize_ue4m3(B, K, mse, p, grid_out, s);
    case kUE5M3: return launch_quantize_ue5m3(B, K, mse, p, grid_out, s);
    default: return cudaErrorInvalidValue;
    }
}

namespace {

template <int K>
cudaError_t run_amax(const AmaxParams& p, cudaStream_t s, bool pdl)
{
    auto kern = amax_kernel<K>;
    const int64_t tiles = p.tile0[p.count];
    const int grid = grid_for((const void*)kern, ring_smem_bytes<K>(), (tiles + kWarps - 1) / kWarps);
    if (pdl) return launch_pdl(kern, grid, kThreads, ring_smem_bytes<K>(), s, p);
    kern<<<grid, kThreads, ring_smem_bytes<K>(), s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_amax_zero(const AmaxParams& p, cudaStream_t s)
{
    amax_zero_kernel<<<1, kAmaxBatch, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_amax(int K, const AmaxParams& p, cudaStream_t s, bool pdl)
{
    switch (K) {
    case 0: return run_amax<0>(p, s, pdl);
    case 16: return run_amax<16>(p, s, pdl);
    case 32: return run_amax<32>(p, s, pdl);
    case 128: return run_amax<128>(p, s, pdl);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace fp4q
