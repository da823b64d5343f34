// fp4q_launch.h -- host-side launchers shared by the C ABI (internal linkage).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp4q {

struct QuantParams;
struct QuantBatchParams;
struct AmaxParams;
struct DequantParams;
struct MseParams;

// Opt a kernel in to `smem` bytes of dynamic shared memory (once per kernel
// and device) and return how many of its CTAs fit on the device at once.
int resident_ctas(const void* kernel, int smem, int threads = 256);

// Device address of the library's fault word on the current device (looked up
// once per device): the tensor-core kernels set it to 1 when a bounded wait on
// the tensor cores gives up instead of hanging.
unsigned int* device_fault_word();

// Grid for a grid-stride kernel: min(ctas_needed, resident CTAs), at least 1.
int grid_for(const void* kernel, int smem, int64_t ctas_needed, int threads = 256);

// CTAs a ring kernel needs for n elements (one 32-unit tile per warp).
int64_t ring_ctas_needed(int64_t n, int ept);

// Each returns cudaSuccess or the launch error; an unsupported (fmt, B, K)
// combination returns cudaErrorInvalidValue before launching anything.
// launch_quantize with mse = true writes per-CTA partials (grid <= max_grid).
cudaError_t launch_quantize(int fmt, int B, int K, bool mse, const QuantParams& p, int* grid_out,
                            cudaStream_t s);
cudaError_t launch_quantize_e8m0(int B, int K, bool mse, const QuantParams& p, int* grid_out, cudaStream_t s);
cudaError_t launch_quantize_ue4m3(int B, int K, bool mse, const QuantParams& p, int* grid_out, cudaStream_t s);
cudaError_t launch_quantize_ue5m3(int B, int K, bool mse, const QuantParams& p, int* grid_out, cudaStream_t s);
// The batched fused quantizer (MXFP4 block 32, NVFP4 block 16); other blocks: cudaErrorInvalidValue.
cudaError_t launch_quantize_batch_e8m0(int B, int K, const QuantBatchParams& p, cudaStream_t s);
cudaError_t launch_quantize_batch_ue4m3(int B, int K, const QuantBatchParams& p, cudaStream_t s);
// pdl: launch with programmatic dependent launch (never right after the memset
// that zeroes the maximum's slot, which must complete first).
// Quantize with MSE-optimised block scales (p.below / p.above candidate codes).
cudaError_t launch_quantize_search(int fmt, int B, int K, const QuantParams& p, cudaStream_t s);
cudaError_t launch_amax(int K, const AmaxParams& p, cudaStream_t s, bool pdl);
cudaError_t launch_amax_zero(const AmaxParams& p, cudaStream_t s);
// Outlier statistics: zeroes the histogram (workspace), stats and col_absmax,
// then one histogram pass over x and a one-CTA scan.
cudaError_t launch_outlier_stats(const uint16_t* x, int64_t rows, int64_t cols, double p, float* stats,
                                 float* col_absmax, void* workspace, cudaStream_t s);
cudaError_t launch_dequantize(int B, int K, bool f32out, const DequantParams& p, cudaStream_t s);
// MSE-optimised per-tensor scale: reads the tensor maximum from workspace + 16
// (written by the amax pass), counter at workspace + 0 (zero at launch).
cudaError_t launch_gscale_search(const uint16_t* x, int64_t n, int fmt, int block, int rot, float c_hi, float c_lo,
                                 int below, int above, float* gscale, double* errors, void* workspace, cudaStream_t s);
size_t gscale_workspace_bytes();
cudaError_t launch_block_mse(int B, int K, const MseParams& p, int* grid_out, cudaStream_t s);

// Launch of a streaming kernel with programmatic dependent launch allowed: the
// grid may be scheduled while the stream's previous kernel drains, and every
// such kernel executes griddepcontrol.wait (pdl_wait) before it touches global
// memory, so it observes everything the stream ordered before it exactly as
// with a plain launch; only launch and scheduling latency overlap.
template <typename P>
inline cudaError_t launch_pdl(void (*kernel)(P), int grid, int threads, int smem, cudaStream_t s, const P& p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Upper bound on the CTAs of any kernel that writes per-CTA partials, and the
// number of partial slots (4 doubles each) a workspace must hold for n elements.
constexpr int kMaxPartialCtas = 4096;
constexpr int64_t kElemsPerPartial = 4096;
inline int64_t partial_slots(int64_t n)
{
    int64_t s = (n + kElemsPerPartial - 1) / kElemsPerPartial;
    if (s < 1) s = 1;
    return s < kMaxPartialCtas ? s : kMaxPartialCtas;
}

}  // namespace fp4q
