// fp4q_api.cu -- the C ABI of libfp4q.so: argument checks, then stream-ordered
// launches.  Nothing here allocates device memory or synchronizes.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fp4q.h"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace {

using namespace fp4q;

constexpr int kAbiVersion = 1;

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Shape / format checks common to every tensor entry point.  On success *n is
// rows * cols.
int check_shape(int64_t rows, int64_t cols, int fmt, int block, int rot, int64_t* n)
{
    if (rows < 0 || cols < 0) return FP4Q_ERR_SHAPE;
    if (fmt != FP4Q_SCALE_E8M0 && fmt != FP4Q_SCALE_UE4M3 && fmt != FP4Q_SCALE_UE5M3)
        return FP4Q_ERR_UNSUPPORTED;
    if (!is_pow2(block) || block < 8 || block > 256) return FP4Q_ERR_UNSUPPORTED;
    if (rot != 0 && rot != 16 && rot != 32 && rot != 128) return FP4Q_ERR_UNSUPPORTED;
    if (cols % block != 0) return FP4Q_ERR_SHAPE;
    if (rot != 0 && cols % rot != 0) return FP4Q_ERR_SHAPE;
    if (cols != 0 && rows > INT64_MAX / 4 / cols) return FP4Q_ERR_SHAPE;
    *n = rows * cols;
    return FP4Q_OK;
}

// 1/sqrt(k) in fp64, split into an fp32 head and an fp32 tail.
void rotation_constants(int rot, float* hi, float* lo)
{
    if (rot == 0) {
        *hi = 1.0f;
        *lo = 0.0f;
        return;
    }
    const double c = 1.0 / std::sqrt((double)rot);
    *hi = (float)c;
    *lo = (float)(c - (double)*hi);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA; }

// MSE workspace: a 16-byte slot whose first word is the completion counter of
// the in-kernel reduction (at a fixed place, so one workspace serves tensors of
// any size), then partial_slots(n) rows of 4 doubles.
constexpr size_t kCounterBytes = 16;
unsigned int* mse_counter(void* workspace) { return static_cast<unsigned int*>(workspace); }
double* mse_partials(void* workspace)
{
    return reinterpret_cast<double*>(static_cast<char*>(workspace) + kCounterBytes);
}

bool valid_gmode(int gmode)
{
    return gmode == FP4Q_GLOBAL_NONE || gmode == FP4Q_GLOBAL_COMPUTE || gmode == FP4Q_GLOBAL_GIVEN ||
           gmode == FP4Q_GLOBAL_FROM_AMAX;
}

// Per-tensor scale source of the quantize kernels for gmode: G itself (GIVEN,
// and COMPUTE after the amax pass), or the tensor maximum in gscale[0] with G
// written to gscale[1] (FROM_AMAX).
void set_global(int gmode, float* gscale, const float** gsrc, float** gdst)
{
    *gsrc = gmode == FP4Q_GLOBAL_NONE ? nullptr : gscale;
    *gdst = gmode == FP4Q_GLOBAL_FROM_AMAX ? gscale + 1 : nullptr;
}

// *dst = max(*dst, amax(|y|)) (fp32 bits, atomicMax: non-negative floats order
// as integers); with `zero` the slot is cleared first.
cudaError_t enqueue_amax(const void* x, int64_t n, int rot, float* dst, cudaStream_t s, bool zero = true)
{
    if (zero) {
        cudaError_t e = cudaMemsetAsync(dst, 0, sizeof(float), s);
        if (e != cudaSuccess) return e;
    }
    if (n == 0) return cudaSuccess;
    AmaxParams ap{};
    ap.count = 1;
    ap.x[0] = static_cast<const uint16_t*>(x);
    ap.n[0] = n;
    ap.tile0[0] = 0;
    ap.tile0[1] = (n + kAmaxTileElems - 1) / kAmaxTileElems;
    ap.amax_bits[0] = reinterpret_cast<unsigned int*>(dst);
    rotation_constants(rot, &ap.c_hi, &ap.c_lo);
    return launch_amax(rot, ap, s, !zero);
}

// ---- fixed scratch of fp4q_block_mse_noalloc
// Per-CTA MSE partials for callers that cannot allocate a workspace: one
// static device buffer per device, 4096 slots of 4 doubles (128 KiB), which is
// the most partial slots any launch uses (the MSE kernel caps its grid there),
// followed by the completion counter (zero at load, left zero by every call).
constexpr int kNoAllocSlots = kMaxPartialCtas;
static __device__ __align__(256) double g_noalloc_partials[kNoAllocSlots * 4 + 2];   // + completion counter

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
double* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_partials on the current device, looked up with
// cudaGetSymbolAddress the first time each device is seen.
int noalloc_partials_for_current_device(double** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP4Q_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return FP4Q_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_partials) != cudaSuccess || !p) return FP4Q_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<double*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return FP4Q_OK;
}

// fp4q_quantize_mse, with the dequantized values written to y (bf16) when y is set.
int quantize_mse_impl(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int gmode,
                      uint8_t* codes, uint8_t* scales, float* gscale, void* y, float* block_mse, double* terms,
                      void* workspace, size_t ws_bytes, void* stream)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, fmt, block, rot, &n);
    if (st) return st;
    if (!valid_gmode(gmode)) return FP4Q_ERR_UNSUPPORTED;
    if (fmt == FP4Q_SCALE_E8M0 && gmode != FP4Q_GLOBAL_NONE) return FP4Q_ERR_UNSUPPORTED;
    if (gmode != FP4Q_GLOBAL_NONE) {
        if (!gscale) return FP4Q_ERR_NULL;
        if (!aligned(gscale, 4)) return FP4Q_ERR_ALIGN;
    }
    if (!terms || !workspace) return FP4Q_ERR_NULL;
    if (!aligned(terms, 8) || !aligned(workspace, 8)) return FP4Q_ERR_ALIGN;
    if (n > 0) {
        if (!x || !codes || !scales) return FP4Q_ERR_NULL;
        if (!aligned(x, 32) || !aligned(codes, 32) || !aligned(scales, 16)) return FP4Q_ERR_ALIGN;
        if (y && !aligned(y, 32)) return FP4Q_ERR_ALIGN;
    }
    if (block_mse && !aligned(block_mse, 16)) return FP4Q_ERR_ALIGN;
    if (ws_bytes < fp4q_block_mse_workspace_size(rows, cols, block)) return FP4Q_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    if (gmode == FP4Q_GLOBAL_COMPUTE) {
        cudaError_t e = enqueue_amax(x, n, rot, gscale, s);
        if (e != cudaSuccess) return FP4Q_ERR_CUDA;
        global_scale_kernel<<<1, 1, 0, s>>>(gscale, gscale);
        if (cudaGetLastError() != cudaSuccess) return FP4Q_ERR_CUDA;
    }
    if (n == 0) {
        if (gmode == FP4Q_GLOBAL_FROM_AMAX) {
            global_scale_kernel<<<1, 1, 0, s>>>(gscale, gscale + 1);
            if (cudaGetLastError() != cudaSuccess) return FP4Q_ERR_CUDA;
        }
        return cuda_status(cudaMemsetAsync(terms, 0, 4 * sizeof(double), s));
    }
    QuantParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.n = n;
    p.codes = codes;
    p.scales = scales;
    set_global(gmode, gscale, &p.gsrc, &p.gdst);
    p.block_mse = block_mse;
    p.partials = mse_partials(workspace);
    p.done = mse_counter(workspace);
    p.terms = terms;
    p.y = static_cast<uint16_t*>(y);
    rotation_constants(rot, &p.c_hi, &p.c_lo);
    int grid = 0;
    return cuda_status(launch_quantize(fmt, block, rot, true, p, &grid, s));
}

}  // namespace

extern "C" {

int fp4q_version(void) { return kAbiVersion; }

int fp4q_device_fault(unsigned int* fault_out, int clear)
{
    if (!fault_out) return FP4Q_ERR_NULL;
    unsigned int* word = device_fault_word();
    if (!word) return FP4Q_ERR_CUDA;
    if (cudaMemcpy(fault_out, word, sizeof(unsigned int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    if (clear && cudaMemset(word, 0, sizeof(unsigned int)) != cudaSuccess) return FP4Q_ERR_CUDA;
    if (clear && cudaDeviceSynchronize() != cudaSuccess) return FP4Q_ERR_CUDA;
    return FP4Q_OK;
}

const char* fp4q_status_string(int status)
{
    switch (status) {
    case FP4Q_OK: return "ok";
    case FP4Q_ERR_NULL: return "a required pointer is NULL";
    case FP4Q_ERR_SHAPE: return "bad shape: negative size, or cols not a multiple of block / rot";
    case FP4Q_ERR_ALIGN: return "misaligned pointer (bf16 tensors and codes: 32 B; scales: 16 B)";
    case FP4Q_ERR_UNSUPPORTED: return "unsupported format, block size, rotation or scale mode";
    case FP4Q_ERR_CUDA: return "CUDA launch or runtime error";
    case FP4Q_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
    }
}

// fp4q_quantize and fp4q_quantize_search: the max rule, or (search) the
// scale search over below / above neighbouring codes.
static int quantize_impl(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int gmode,
                         uint8_t* codes, uint8_t* scales, float* gscale, bool search, int below, int above,
                         void* stream, bool mma_layout = false)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, fmt, block, rot, &n);
    if (st) return st;
    if (mma_layout && !((fmt == FP4Q_SCALE_E8M0 && block == 32) || (fmt == FP4Q_SCALE_UE4M3 && block == 16)))
        return FP4Q_ERR_UNSUPPORTED;
    if (!valid_gmode(gmode)) return FP4Q_ERR_UNSUPPORTED;
    if (fmt == FP4Q_SCALE_E8M0 && gmode != FP4Q_GLOBAL_NONE) return FP4Q_ERR_UNSUPPORTED;
    if (gmode != FP4Q_GLOBAL_NONE) {
        if (!gscale) return FP4Q_ERR_NULL;
        if (!aligned(gscale, 4)) return FP4Q_ERR_ALIGN;
    }
    if (n > 0) {
        if (!x || !codes || !scales) return FP4Q_ERR_NULL;
        if (!aligned(x, 32) || !aligned(codes, 32) || !aligned(scales, 16)) return FP4Q_ERR_ALIGN;
    }
    cudaStream_t s = as_stream(stream);
    if (gmode == FP4Q_GLOBAL_COMPUTE) {
        cudaError_t e = enqueue_amax(x, n, rot, gscale, s);
        if (e != cudaSuccess) return FP4Q_ERR_CUDA;
        global_scale_kernel<<<1, 1, 0, s>>>(gscale, gscale);
        if (cudaGetLastError() != cudaSuccess) return FP4Q_ERR_CUDA;
    }
    if (n == 0) {
        if (gmode == FP4Q_GLOBAL_FROM_AMAX) {
            global_scale_kernel<<<1, 1, 0, s>>>(gscale, gscale + 1);
            return cuda_status(cudaGetLastError());
        }
        return FP4Q_OK;
    }
    QuantParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.n = n;
    p.codes = codes;
    p.scales = scales;
    set_global(gmode, gscale, &p.gsrc, &p.gdst);
    rotation_constants(rot, &p.c_hi, &p.c_lo);
    if (mma_layout) {
        p.sf_cols = cols / block;
        p.sf_kt = (p.sf_cols + 3) / 4;
    }
    if (search) {
        p.below = below;
        p.above = above;
        return cuda_status(launch_quantize_search(fmt, block, rot, p, s));
    }
    return cuda_status(launch_quantize(fmt, block, rot, false, p, nullptr, s));
}

int fp4q_quantize(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int gmode,
                  uint8_t* codes, uint8_t* scales, float* gscale, void* stream)
{
    return quantize_impl(x, rows, cols, fmt, block, rot, gmode, codes, scales, gscale, false, 0, 0, stream);
}

size_t fp4q_global_scale_search_workspace_size(void) { return gscale_workspace_bytes(); }

int fp4q_global_scale_search(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int below,
                             int above, float* gscale, double* errors, void* workspace, size_t ws_bytes,
                             void* stream)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, fmt, block, rot, &n);
    if (st) return st;
    if (fmt == FP4Q_SCALE_E8M0) return FP4Q_ERR_UNSUPPORTED;
    if (below < 0 || below > 8 || above < 0 || above > 15) return FP4Q_ERR_UNSUPPORTED;
    if (!gscale || !workspace) return FP4Q_ERR_NULL;
    if (!aligned(gscale, 4) || !aligned(workspace, 16) || (errors && !aligned(errors, 8))) return FP4Q_ERR_ALIGN;
    if (ws_bytes < gscale_workspace_bytes()) return FP4Q_ERR_WORKSPACE;
    if (n > 0 && !x) return FP4Q_ERR_NULL;
    if (n > 0 && !aligned(x, 32)) return FP4Q_ERR_ALIGN;
    cudaStream_t s = as_stream(stream);
    if (n == 0) {
        // an empty tensor: G0 = 1 is the only sensible scale; every candidate's error is 0
        if (errors && cudaMemsetAsync(errors, 0, (size_t)(below + above + 1) * sizeof(double), s) != cudaSuccess)
            return FP4Q_ERR_CUDA;
        if (cudaMemsetAsync(static_cast<uint8_t*>(workspace) + 16, 0, 4, s) != cudaSuccess) return FP4Q_ERR_CUDA;
        global_scale_kernel<<<1, 1, 0, s>>>(static_cast<const float*>(workspace) + 4, gscale);
        return cuda_status(cudaGetLastError());
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (cudaMemsetAsync(ws, 0, 16, s) != cudaSuccess) return FP4Q_ERR_CUDA;          // completion counter
    cudaError_t e = enqueue_amax(x, n, rot, reinterpret_cast<float*>(ws + 16), s);  // the tensor maximum
    if (e != cudaSuccess) return FP4Q_ERR_CUDA;
    float c_hi = 0.0f, c_lo = 0.0f;
    rotation_constants(rot, &c_hi, &c_lo);
    return cuda_status(launch_gscale_search(static_cast<const uint16_t*>(x), n, fmt, block, rot, c_hi, c_lo, below,
                                            above, gscale, errors, workspace, s));
}

size_t fp4q_mma_scales_size(int64_t rows, int64_t cols, int block)
{
    if (rows <= 0 || cols <= 0 || block <= 0) return 0;
    const int64_t sf_cols = cols / block;
    return (size_t)(((rows + 127) / 128) * ((sf_cols + 3) / 4) * 512);
}

int fp4q_quantize_mma(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int gmode,
                      uint8_t* codes, uint8_t* scales_mma, float* gscale, void* stream)
{
    return quantize_impl(x, rows, cols, fmt, block, rot, gmode, codes, scales_mma, gscale, false, 0, 0, stream,
                         true);
}

int fp4q_quantize_search(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int gmode,
                         int below, int above, uint8_t* codes, uint8_t* scales, float* gscale, void* stream)
{
    if (below < 0 || below > FP4Q_SEARCH_MAX || above < 0 || above > FP4Q_SEARCH_MAX) return FP4Q_ERR_UNSUPPORTED;
    return quantize_impl(x, rows, cols, fmt, block, rot, gmode, codes, scales, gscale, true, below, above, stream);
}

int fp4q_quantize_mse(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int gmode,
                      uint8_t* codes, uint8_t* scales, float* gscale, float* block_mse, double* terms,
                      void* workspace, size_t ws_bytes, void* stream)
{
    return quantize_mse_impl(x, rows, cols, fmt, block, rot, gmode, codes, scales, gscale, nullptr, block_mse,
                             terms, workspace, ws_bytes, stream);
}

int fp4q_quantize_mse_dequantize(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                                 int gmode, uint8_t* codes, uint8_t* scales, float* gscale, void* y,
                                 float* block_mse, double* terms, void* workspace, size_t ws_bytes, void* stream)
{
    if (rows > 0 && cols > 0 && !y) return FP4Q_ERR_NULL;
    return quantize_mse_impl(x, rows, cols, fmt, block, rot, gmode, codes, scales, gscale, y, block_mse, terms,
                             workspace, ws_bytes, stream);
}

// Per-tensor slice of the batched quantizer's workspace: the completion counter,
// then kMaxPartialCtas partial slots of 4 doubles.
constexpr size_t kBatchSliceBytes = kCounterBytes + (size_t)kMaxPartialCtas * 4 * sizeof(double);

size_t fp4q_quantize_batch_workspace_size(int count)
{
    return count > 0 ? (size_t)count * kBatchSliceBytes : 0;
}

int fp4q_quantize_mse_dequantize_batched(int count, const fp4q_tensor* tensors, int fmt, int block, int rot,
                                         int gmode, void* workspace, size_t ws_bytes, void* stream)
{
    if (count < 0) return FP4Q_ERR_SHAPE;
    if (count == 0) return FP4Q_OK;
    if (!tensors || !workspace) return FP4Q_ERR_NULL;
    if (!((fmt == FP4Q_SCALE_E8M0 && block == 32) || (fmt == FP4Q_SCALE_UE4M3 && block == 16)))
        return FP4Q_ERR_UNSUPPORTED;
    if (!valid_gmode(gmode)) return FP4Q_ERR_UNSUPPORTED;
    if (fmt == FP4Q_SCALE_E8M0 && gmode != FP4Q_GLOBAL_NONE) return FP4Q_ERR_UNSUPPORTED;
    if (!aligned(workspace, 8)) return FP4Q_ERR_ALIGN;
    if (ws_bytes < fp4q_quantize_batch_workspace_size(count)) return FP4Q_ERR_WORKSPACE;
    for (int i = 0; i < count; ++i) {                  // every tensor checked before anything is enqueued
        const fp4q_tensor& t = tensors[i];
        int64_t n = 0;
        int st = check_shape(t.rows, t.cols, fmt, block, rot, &n);
        if (st) return st;
        if (!t.terms) return FP4Q_ERR_NULL;
        if (!aligned(t.terms, 8)) return FP4Q_ERR_ALIGN;
        if (gmode != FP4Q_GLOBAL_NONE) {
            if (!t.gscale) return FP4Q_ERR_NULL;
            if (!aligned(t.gscale, 4)) return FP4Q_ERR_ALIGN;
        }
        if (n > 0) {
            if (!t.x || !t.codes || !t.scales || !t.y) return FP4Q_ERR_NULL;
            if (!aligned(t.x, 32) || !aligned(t.codes, 32) || !aligned(t.scales, 16) || !aligned(t.y, 32))
                return FP4Q_ERR_ALIGN;
        }
        if (t.block_mse && !aligned(t.block_mse, 16)) return FP4Q_ERR_ALIGN;
        if (n > (int64_t)(INT32_MAX / kQuantBatch) * kAmaxTileElems) return FP4Q_ERR_SHAPE;   // tile indices fit 32 bits
    }
    cudaStream_t s = as_stream(stream);
    if (gmode == FP4Q_GLOBAL_COMPUTE) {
        // the tensors' maxima, then G = amax / 2688 in place; the quantizer reads G as given
        for (int i = 0; i < count; ++i) {
            const fp4q_tensor& t = tensors[i];
            cudaError_t e = enqueue_amax(t.x, t.rows * t.cols, rot, t.gscale, s);
            if (e == cudaSuccess) {
                global_scale_kernel<<<1, 1, 0, s>>>(t.gscale, t.gscale);
                e = cudaGetLastError();
            }
            if (e != cudaSuccess) return FP4Q_ERR_CUDA;
        }
    }
    char* ws = static_cast<char*>(workspace);
    for (int c0 = 0; c0 < count; c0 += kQuantBatch) {
        QuantBatchParams bp{};
        bp.count = count - c0 < kQuantBatch ? count - c0 : kQuantBatch;
        bp.tile0[0] = 0;
        for (int j = 0; j < bp.count; ++j) {
            const fp4q_tensor& t = tensors[c0 + j];
            QuantParams& q = bp.t[j];
            q.x = static_cast<const uint16_t*>(t.x);
            q.n = t.rows * t.cols;
            q.codes = t.codes;
            q.scales = t.scales;
            set_global(gmode == FP4Q_GLOBAL_COMPUTE ? FP4Q_GLOBAL_GIVEN : gmode, t.gscale, &q.gsrc, &q.gdst);
            q.block_mse = t.block_mse;
            void* slice = ws + (size_t)(c0 + j) * kBatchSliceBytes;
            q.partials = mse_partials(slice);
            q.done = mse_counter(slice);
            q.terms = t.terms;
            q.y = static_cast<uint16_t*>(t.y);
            rotation_constants(rot, &q.c_hi, &q.c_lo);
            bp.tile0[j + 1] = bp.tile0[j] + (int32_t)((q.n + kAmaxTileElems - 1) / kAmaxTileElems);
        }
        cudaError_t e = fmt == FP4Q_SCALE_E8M0 ? launch_quantize_batch_e8m0(block, rot, bp, s)
                                               : launch_quantize_batch_ue4m3(block, rot, bp, s);
        if (e != cudaSuccess) return FP4Q_ERR_CUDA;
    }
    return FP4Q_OK;
}

int fp4q_tensor_amax(const void* x, int64_t rows, int64_t cols, int rot, float* amax, void* stream)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, FP4Q_SCALE_E8M0, 8, rot, &n);
    if (st) return st;
    if (!amax || (n > 0 && !x)) return FP4Q_ERR_NULL;
    if (!aligned(amax, 4) || (n > 0 && !aligned(x, 32))) return FP4Q_ERR_ALIGN;
    return cuda_status(enqueue_amax(x, n, rot, amax, as_stream(stream)));
}

int fp4q_tensor_amax_accumulate(const void* x, int64_t rows, int64_t cols, int rot, float* amax, void* stream)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, FP4Q_SCALE_E8M0, 8, rot, &n);
    if (st) return st;
    if (!amax || (n > 0 && !x)) return FP4Q_ERR_NULL;
    if (!aligned(amax, 4) || (n > 0 && !aligned(x, 32))) return FP4Q_ERR_ALIGN;
    return cuda_status(enqueue_amax(x, n, rot, amax, as_stream(stream), false));
}

int fp4q_tensor_amax_batched(int count, const void* const* xs, const int64_t* rows, const int64_t* cols, int rot,
                             float* const* amax, int accumulate, void* stream)
{
    if (count < 0) return FP4Q_ERR_SHAPE;
    if (count == 0) return FP4Q_OK;
    if (!xs || !rows || !cols || !amax) return FP4Q_ERR_NULL;
    for (int i = 0; i < count; ++i) {                 // every tensor checked before anything is enqueued
        int64_t n = 0;
        int st = check_shape(rows[i], cols[i], FP4Q_SCALE_E8M0, 8, rot, &n);
        if (st) return st;
        if (!amax[i] || (n > 0 && !xs[i])) return FP4Q_ERR_NULL;
        if (!aligned(amax[i], 4) || (n > 0 && !aligned(xs[i], 32))) return FP4Q_ERR_ALIGN;
    }
    cudaStream_t s = as_stream(stream);
    for (int c0 = 0; c0 < count; c0 += kAmaxBatch) {
        AmaxParams ap{};
        ap.count = count - c0 < kAmaxBatch ? count - c0 : kAmaxBatch;
        rotation_constants(rot, &ap.c_hi, &ap.c_lo);
        ap.tile0[0] = 0;
        for (int j = 0; j < ap.count; ++j) {
            ap.x[j] = static_cast<const uint16_t*>(xs[c0 + j]);
            ap.n[j] = rows[c0 + j] * cols[c0 + j];
            ap.tile0[j + 1] = ap.tile0[j] + (ap.n[j] + kAmaxTileElems - 1) / kAmaxTileElems;
            ap.amax_bits[j] = reinterpret_cast<unsigned int*>(amax[c0 + j]);
        }
        cudaError_t e = cudaSuccess;
        if (!accumulate) e = launch_amax_zero(ap, s);
        if (e == cudaSuccess && ap.tile0[ap.count] > 0) e = launch_amax(rot, ap, s, true);
        if (e != cudaSuccess) return FP4Q_ERR_CUDA;
    }
    return FP4Q_OK;
}

int fp4q_global_scale(const float* amax, float* gscale, void* stream)
{
    if (!amax || !gscale) return FP4Q_ERR_NULL;
    if (!aligned(amax, 4) || !aligned(gscale, 4)) return FP4Q_ERR_ALIGN;
    global_scale_kernel<<<1, 1, 0, as_stream(stream)>>>(amax, gscale);
    return cuda_status(cudaGetLastError());
}

int fp4q_dequantize(const uint8_t* codes, const uint8_t* scales, const float* gscale, int64_t rows,
                    int64_t cols, int fmt, int block, int rot, int out_dtype, void* y, void* stream)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, fmt, block, rot, &n);
    if (st) return st;
    if (out_dtype != FP4Q_OUT_BF16 && out_dtype != FP4Q_OUT_F32) return FP4Q_ERR_UNSUPPORTED;
    if (gscale && !aligned(gscale, 4)) return FP4Q_ERR_ALIGN;
    if (n == 0) return FP4Q_OK;
    if (!codes || !scales || !y) return FP4Q_ERR_NULL;
    if (!aligned(codes, 32) || !aligned(scales, 16) || !aligned(y, 32)) return FP4Q_ERR_ALIGN;
    DequantParams p{};
    p.codes = codes;
    p.scales = scales;
    p.gsrc = gscale;
    p.n = n;
    p.fmt = fmt;
    p.y = y;
    rotation_constants(rot, &p.c_hi, &p.c_lo);
    return cuda_status(launch_dequantize(block, rot, out_dtype == FP4Q_OUT_F32, p, as_stream(stream)));
}

size_t fp4q_outlier_stats_workspace_size(void) { return (size_t)FP4Q_OUTLIER_WS_BYTES; }

int fp4q_outlier_stats(const void* x, int64_t rows, int64_t cols, double p, float* stats, float* col_absmax,
                       void* workspace, size_t ws_bytes, void* stream)
{
    if (rows < 0 || cols < 0 || cols % 8 != 0) return FP4Q_ERR_SHAPE;
    if (cols != 0 && rows > INT64_MAX / 4 / cols) return FP4Q_ERR_SHAPE;
    if (!(p > 0.0 && p <= 1.0)) return FP4Q_ERR_UNSUPPORTED;
    if (!stats || !workspace) return FP4Q_ERR_NULL;
    if (ws_bytes < (size_t)FP4Q_OUTLIER_WS_BYTES) return FP4Q_ERR_WORKSPACE;
    if (!aligned(stats, 4) || !aligned(workspace, 8) || (col_absmax && !aligned(col_absmax, 4)))
        return FP4Q_ERR_ALIGN;
    const int64_t n = rows * cols;
    if (n > 0) {
        if (!x) return FP4Q_ERR_NULL;
        if (!aligned(x, 16)) return FP4Q_ERR_ALIGN;
    }
    return cuda_status(launch_outlier_stats(static_cast<const uint16_t*>(x), rows, cols, p, stats, col_absmax,
                                            workspace, as_stream(stream)));
}

size_t fp4q_block_mse_workspace_size(int64_t rows, int64_t cols, int block)
{
    (void)block;
    if (rows < 0 || cols < 0) return 0;
    if (cols != 0 && rows > INT64_MAX / 4 / cols) return 0;
    return (size_t)partial_slots(rows * cols) * 4 * sizeof(double) + kCounterBytes;
}

int fp4q_block_mse(const void* x, const uint8_t* codes, const uint8_t* scales, const float* gscale,
                   int64_t rows, int64_t cols, int fmt, int block, int rot, float* block_mse,
                   double* terms, void* workspace, size_t ws_bytes, void* stream)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, fmt, block, rot, &n);
    if (st) return st;
    if (!terms || !workspace) return FP4Q_ERR_NULL;
    if (n > 0 && (!x || !codes || !scales)) return FP4Q_ERR_NULL;
    if (!aligned(terms, 8) || !aligned(workspace, 8)) return FP4Q_ERR_ALIGN;
    if (gscale && !aligned(gscale, 4)) return FP4Q_ERR_ALIGN;
    if (n > 0 && (!aligned(x, 32) || !aligned(codes, 32) || !aligned(scales, 16)))
        return FP4Q_ERR_ALIGN;
    if (block_mse && !aligned(block_mse, 16)) return FP4Q_ERR_ALIGN;
    if (ws_bytes < fp4q_block_mse_workspace_size(rows, cols, block)) return FP4Q_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    if (n == 0) return cuda_status(cudaMemsetAsync(terms, 0, 4 * sizeof(double), s));
    MseParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.codes = codes;
    p.scales = scales;
    p.gsrc = gscale;
    p.n = n;
    p.fmt = fmt;
    p.block_mse = block_mse;
    p.partials = mse_partials(workspace);
    p.done = mse_counter(workspace);
    p.terms = terms;
    rotation_constants(rot, &p.c_hi, &p.c_lo);
    int grid = 0;
    return cuda_status(launch_block_mse(block, rot, p, &grid, s));
}

int fp4q_e2m1_encode_f32(const float* r, int64_t n, uint8_t* packed, void* stream)
{
    if (n < 0 || (n & 1)) return FP4Q_ERR_SHAPE;
    if (n == 0) return FP4Q_OK;
    if (!r || !packed) return FP4Q_ERR_NULL;
    if (!aligned(r, 4) || !aligned(packed, 4)) return FP4Q_ERR_ALIGN;
    const int64_t work = (n + 7) / 8;
    int grid = grid_for((const void*)e2m1_encode_kernel, 0, (work + kThreads - 1) / kThreads);
    e2m1_encode_kernel<<<grid, kThreads, 0, as_stream(stream)>>>(r, n, packed);
    return cuda_status(cudaGetLastError());
}

int fp4q_scale_encode_f32(const float* s, int64_t n, int fmt, uint8_t* codes, void* stream)
{
    if (n < 0) return FP4Q_ERR_SHAPE;
    if (fmt != FP4Q_SCALE_E8M0 && fmt != FP4Q_SCALE_UE4M3 && fmt != FP4Q_SCALE_UE5M3)
        return FP4Q_ERR_UNSUPPORTED;
    if (n == 0) return FP4Q_OK;
    if (!s || !codes) return FP4Q_ERR_NULL;
    if (!aligned(s, 4) || !aligned(codes, 4)) return FP4Q_ERR_ALIGN;
    int grid = grid_for((const void*)scale_encode_kernel, 0, (n + kThreads - 1) / kThreads);
    scale_encode_kernel<<<grid, kThreads, 0, as_stream(stream)>>>(s, n, fmt, codes);
    return cuda_status(cudaGetLastError());
}

int fp4q_block_mse_noalloc(const void* x, const uint8_t* codes, const uint8_t* scales, const float* gscale,
                           int64_t rows, int64_t cols, int fmt, int block, int rot, float* block_mse,
                           double* terms, void* stream)
{
    int64_t n = 0;
    int st = check_shape(rows, cols, fmt, block, rot, &n);
    if (st) return st;
    if (!terms) return FP4Q_ERR_NULL;
    if (n > 0 && (!x || !codes || !scales)) return FP4Q_ERR_NULL;
    if (!aligned(terms, 8)) return FP4Q_ERR_ALIGN;
    if (gscale && !aligned(gscale, 4)) return FP4Q_ERR_ALIGN;
    if (n > 0 && (!aligned(x, 32) || !aligned(codes, 32) || !aligned(scales, 16)))
        return FP4Q_ERR_ALIGN;
    if (block_mse && !aligned(block_mse, 16)) return FP4Q_ERR_ALIGN;
    if (partial_slots(n) > kNoAllocSlots) return FP4Q_ERR_WORKSPACE;
    double* partials = nullptr;
    st = noalloc_partials_for_current_device(&partials);
    if (st) return st;
    cudaStream_t s = as_stream(stream);
    if (n == 0) return cuda_status(cudaMemsetAsync(terms, 0, 4 * sizeof(double), s));
    MseParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.codes = codes;
    p.scales = scales;
    p.gsrc = gscale;
    p.n = n;
    p.fmt = fmt;
    p.block_mse = block_mse;
    p.partials = partials;
    p.done = reinterpret_cast<unsigned int*>(partials + kNoAllocSlots * 4);
    p.terms = terms;
    rotation_constants(rot, &p.c_hi, &p.c_lo);
    // the launch uses at most partial_slots(n) CTAs, checked above to fit the scratch
    int grid = 0;
    return cuda_status(launch_block_mse(block, rot, p, &grid, s));
}

}  // extern "C"
