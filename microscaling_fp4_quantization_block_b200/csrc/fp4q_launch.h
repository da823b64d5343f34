// fp4q_launch.h -- host-side launchers shared by the C ABI (internal linkage).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp4q {

struct QuantParams;
struct AmaxParams;
struct DequantParams;
struct MseParams;

// Grid size for a grid-stride kernel: enough CTAs for the work, at most the
// number that fit on the device at once (occupancy x SM count).
int resident_grid(const void* kernel, int64_t ctas_needed);

// Each returns cudaSuccess or the launch error; an unsupported (fmt, B, K)
// combination returns cudaErrorInvalidValue before launching anything.
cudaError_t launch_quantize(int fmt, int B, int K, const QuantParams& p, cudaStream_t s);
cudaError_t launch_amax(int K, const AmaxParams& p, cudaStream_t s);
cudaError_t launch_dequantize(int B, int K, bool f32out, const DequantParams& p, cudaStream_t s);
cudaError_t launch_block_mse(int B, int K, const MseParams& p, int grid, cudaStream_t s);
int mse_grid(int B, int K, int64_t n);

// Elements one warp-tile covers (32 lanes x units in flight x elements per unit).
constexpr int64_t kTileElems = 2048;
constexpr int kMaxMseCtas = 4096;

}  // namespace fp4q
