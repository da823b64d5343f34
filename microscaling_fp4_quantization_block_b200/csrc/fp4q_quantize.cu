// fp4q_quantize.cu -- launch helpers, format dispatch of quantize, and the amax kernels.
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"
#include "fp4q_tc.cuh"

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

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}
}  // namespace

bool encode_tensor_map_2d(void* map, int elem_bytes, const void* base, uint64_t inner, uint64_t rows,
                          uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, int swizzle)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc || rows == 0 || inner == 0) return false;
    const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(static_cast<CUtensorMap*>(map), dt, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, static_cast<CUtensorMapSwizzle>(swizzle),
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
    int sms = 0, occ = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem);
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
    // the rotation on the tensor cores, 4096-element tiles through a TMA ring of
    // 32-element rows; a tensor whose size is an odd multiple of 16 rotates with
    // the butterfly kernel below
    if constexpr (K == 16 || K == 32) {
        if (p.n % 32 == 0) {
            TcAmaxParams tp;
            memset(&tp, 0, sizeof(tp));
            tp.p = p;
            tp.p.fault = device_fault_word();
            if (tp.p.fault == nullptr) return cudaErrorInvalidDevice;
            if (!encode_tensor_map_2d(&tp.xmap, 2, p.x, tc::KR, (uint64_t)(p.n / tc::KR), 2 * tc::KR, tc::KR,
                                      tc::ROWS, CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
            auto kern = amax_tc_kernel<K>;
            const int64_t tiles = (p.n + tc::TILE_ELEMS - 1) / tc::TILE_ELEMS;
            const int grid = grid_for((const void*)kern, tc::SMEM_BYTES, tiles, tc::THREADS);
            if (pdl) return launch_pdl(kern, grid, tc::THREADS, tc::SMEM_BYTES, s, tp);
            kern<<<grid, tc::THREADS, tc::SMEM_BYTES, s>>>(tp);
            return cudaGetLastError();
        }
    }
    auto kern = amax_kernel<K>;
    const int grid = grid_for((const void*)kern, kRingBytesPerCta, ring_ctas_needed(p.n, EPT));
    if (pdl) return launch_pdl(kern, grid, kThreads, kRingBytesPerCta, s, p);
    kern<<<grid, kThreads, kRingBytesPerCta, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

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
