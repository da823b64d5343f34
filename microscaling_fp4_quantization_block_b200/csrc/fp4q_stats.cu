// fp4q_stats.cu -- activation outlier statistics ("Diagnosing FP4 inference",
// Methodology and Results C: the maximum and the 99.9th percentile of the
// activations, whose ratio separates the down projection from the others).
//
// max |x|, the nearest-rank p-quantile of |x| (the k-th smallest magnitude,
// k = ceil(p n)) and the per-channel maxima of a bf16 [rows][cols] tensor.
// A bf16 magnitude has 2^15 bit patterns, and non-negative bf16 values order
// like their patterns, so a histogram over the patterns gives the quantile
// exactly.
//
// Only the magnitudes near the quantile need counting one by one.  A tensor of
// at least kDirectElems elements is therefore done in three steps:
//  1. a histogram of every s-th row estimates the quantile, and sets a
//     threshold L a safe margin below it;
//  2. the main pass histograms only magnitudes >= L (a few in a thousand for
//     P99.9) and takes every channel maximum; the magnitudes below L are then
//     n minus the histogram's total.  When the sample puts at most 1/64 of
//     the magnitudes at or above L, the main pass is a streaming kernel at
//     full occupancy (the quantizer's cp.async ring, column stripes so that a
//     lane keeps its channels' maxima in registers) that adds each counted
//     magnitude to the global histogram with an atomic (the next launch then
//     sums its 128-bin bucket totals: atomics on the few buckets that hold
//     the top magnitudes would serialise); otherwise a pass with a
//     shared-memory histogram per CTA does it (both launches read a device
//     flag set by the threshold scan);
//  3. if rank k falls among the counted magnitudes the answer is exact;
//     otherwise (L was not below the quantile) a pass gated on a device flag
//     adds the magnitudes below L, and the scan is repeated on the full
//     histogram.
// Smaller tensors take one full histogram pass.
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

constexpr int kBins = 1 << 15;               // bf16 magnitude patterns
constexpr int kBuckets = 256;                 // one per exponent field: 128 mantissa bins each
constexpr int kStatThreads = 1024;
constexpr int kHistSmem = kBins * 4;          // 128 KiB of per-CTA counts
constexpr int64_t kDirectElems = int64_t(1) << 22;
constexpr int64_t kSampleElems = int64_t(1) << 20;   // at least this many in the estimate
constexpr int kMaxSampleStride = 16;

constexpr int kSparseDiv = 64;                // sparse main pass when <= 1/64 of the sample is >= L

struct StatsCtl {
    uint32_t L;          // magnitudes >= L are counted by the main pass
    uint32_t fallback;   // set when the rank lies below L
    uint32_t dense;      // set when the sample puts more than 1/kSparseDiv of the magnitudes at or above L
    uint32_t pad;
};

static_assert(sizeof(StatsCtl) == 16, "the workspace holds 16 bytes of control words");

enum : int { kAllBins = 0, kFromL = 1, kBelowLIfNeeded = 2, kFromLIfDense = 3 };

struct StatsParams {
    const uint16_t* x;
    int64_t rows;              // rows visited: 0, row_step, 2 row_step, ... (rows of them)
    int64_t row_step;
    int64_t g;                 // 16-byte chunks per row (cols / 8)
    int64_t r;                 // visited rows between a thread's consecutive rows
    int64_t T;                 // working threads: g * r
    unsigned long long* hist;  // [kBins] counts
    unsigned long long* buck;  // [kBuckets] totals of hist's 128-bin buckets
    unsigned int* colmax;      // [cols] fp32 bits of the channel maxima (zeroed) or nullptr
    const StatsCtl* ctl;
    int mode;
};

__device__ __forceinline__ uint4 ldg128_stream(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Fold a chunk's 8 magnitudes into this thread's channel maxima (two channels
// per word, packed), and count those in [lo, lo + span).  A chunk whose largest
// magnitude is below lo -- almost every chunk when only the top of the
// distribution is counted -- costs a few packed maxima and one branch.
__device__ __forceinline__ void count_chunk(const uint4& v, uint32_t* sh, uint32_t lo, uint32_t span,
                                            uint32_t (&cmw)[4])
{
    const uint32_t w[4] = {v.x & 0x7fff7fffu, v.y & 0x7fff7fffu, v.z & 0x7fff7fffu, v.w & 0x7fff7fffu};
#pragma unroll
    for (int k = 0; k < 4; ++k) cmw[k] = max_u16x2(cmw[k], w[k]);
    const uint32_t m = max_u16x2(max_u16x2(w[0], w[1]), max_u16x2(w[2], w[3]));
    if (max(m & 0xffffu, m >> 16) < lo) return;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t a = w[k] & 0xffffu, b = w[k] >> 16;
        if (a - lo < span) atomicAdd(sh + a, 1u);
        if (b - lo < span) atomicAdd(sh + b, 1u);
    }
}

// Thread t owns the 8 channels of chunk t % g in visited rows t / g, t / g + r,
// ...: consecutive threads read consecutive 16-byte chunks of a row, and a
// thread's channel maxima stay in registers until the end.
__global__ void __launch_bounds__(kStatThreads, 1) outlier_hist_kernel(StatsParams p)
{
    pdl_wait();
    pdl_release();
    uint32_t lo = 0u, hi = (uint32_t)kBins;
    if (p.mode == kFromL || p.mode == kFromLIfDense) {
        if (p.mode == kFromLIfDense && !p.ctl->dense) {
            // the sparse pass ran: its histogram's bucket totals, 8 buckets per CTA
            // (a thread per bin), written whole (nothing else has touched them)
            if (blockIdx.x >= kBuckets / 8) return;
            __shared__ unsigned long long part[32];
            const int b = (int)blockIdx.x * 8 + (int)(threadIdx.x >> 7);
            unsigned long long c = p.hist[128 * b + (threadIdx.x & 127)];
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) c += __shfl_xor_sync(0xffffffffu, c, d);
            if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
            __syncthreads();
            if ((threadIdx.x & 127) == 0) {
                const int w0 = (int)(threadIdx.x >> 5);
                p.buck[b] = part[w0] + part[w0 + 1] + part[w0 + 2] + part[w0 + 3];
            }
            return;
        }
        lo = p.ctl->L;
    } else if (p.mode == kBelowLIfNeeded) {
        if (!p.ctl->fallback) return;
        hi = p.ctl->L;
    }
    extern __shared__ __align__(16) uint32_t sh_hist[];
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) sh_hist[i] = 0u;
    __syncthreads();
    const uint32_t span = hi - lo;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t cmw[4] = {0u, 0u, 0u, 0u};                           // channel maxima, two per word
    if (tid < p.T) {
        const int64_t c8 = tid % p.g;
        const uint4* base = reinterpret_cast<const uint4*>(p.x) + c8;
        const int64_t stride = p.row_step * p.g;                  // chunks between visited rows
        int64_t j = tid / p.g;
        for (; j + 7 * p.r < p.rows; j += 8 * p.r) {                // 8 loads in flight
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = ldg128_stream(base + (j + u * p.r) * stride);
#pragma unroll
            for (int u = 0; u < 8; ++u) count_chunk(v[u], sh_hist, lo, span, cmw);
        }
        for (; j < p.rows; j += p.r) count_chunk(ldg128_stream(base + j * stride), sh_hist, lo, span, cmw);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) {
        const uint32_t c = sh_hist[i];
        if (c) atomicAdd(p.hist + i, (unsigned long long)c);
    }
    {
        // bucket totals: four threads per bucket, 32 bins each, the bin order
        // rotated by lane so that a warp's shared reads hit 32 different banks
        const int t = threadIdx.x, l = t & 31;
        const uint32_t* b = sh_hist + 32 * t;                   // bins 32 t .. 32 t + 31 = part t % 4 of bucket t / 4
        unsigned long long sum = 0;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) sum += b[(j + l) & 31];
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if ((t & 3) == 0 && sum) atomicAdd(p.buck + (t >> 2), sum);
    }
    if (tid < p.T && p.colmax) {
        unsigned int* dst = p.colmax + 8 * (tid % p.g);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t c = (j & 1) ? cmw[j >> 1] >> 16 : cmw[j >> 1] & 0xffffu;
            if (c) atomicMax(dst + j, c << 16);              // |x| as fp32 bits: orders as integers
        }
    }
}

// ---- the sparse main pass: magnitudes >= L, global atomics, streaming ring
// A tile is 4 rows x 256 channels (512 bytes a row): lane l copies and reads
// the 16-byte chunk of channels 8 l .. 8 l + 7 of each row.  Tiles are numbered
// column block first; when the number of warps is a multiple of the number of
// column blocks (the launch picks such a grid when it can) a warp's column
// block never changes and its lanes' channel maxima stay in registers, else
// they are flushed whenever it does.
constexpr int kTopRows = 4;
using TopRing = Ring<16, kTopRows>;

struct TopParams {
    const uint16_t* x;
    int64_t rows, cols;
    int64_t ncb;                 // 256-channel column blocks
    unsigned long long* hist;
    unsigned int* colmax;        // or nullptr
    const StatsCtl* ctl;
};

// Tile cursor: the warp's tiles advance by n_warps, i.e. by dcb column blocks and
// drg row groups (n_warps = drg * ncb + dcb), with no division per tile.
struct TileCursor {
    int64_t cb, rg;
    __device__ __forceinline__ void step(int64_t dcb, int64_t drg, int64_t ncb)
    {
        cb += dcb;
        rg += drg;
        if (cb >= ncb) {
            cb -= ncb;
            ++rg;
        }
    }
};

// The channel maxima cmw hold, per bf16 half, a value whose magnitude is the
// largest seen (max.xorsign.abs leaves a meaningless sign: the flush masks it).
// Inputs are finite, so the bf16 maximum of magnitudes is the integer maximum of
// their patterns.
__device__ __forceinline__ void count_top(const uint32_t (&w)[4], const TopParams& p, uint32_t lo, uint32_t span,
                                          uint32_t (&cmw)[4])
{
#pragma unroll
    for (int k = 0; k < 4; ++k) cmw[k] = bf16x2_absmax(cmw[k], w[k]);
    const uint32_t m = bf16x2_absmax(bf16x2_absmax(w[0], w[1]), bf16x2_absmax(w[2], w[3])) & 0x7fff7fffu;
    if (max(m & 0xffffu, m >> 16) < lo) return;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t v = ((k & 1) ? w[k >> 1] >> 16 : w[k >> 1]) & 0x7fffu;
        if (v - lo < span) atomicAdd(p.hist + v, 1ull);
    }
}

__global__ void __launch_bounds__(kThreads) outlier_top_kernel(TopParams p)
{
    pdl_wait();
    pdl_release();
    if (p.ctl->dense) return;
    const uint32_t lo = p.ctl->L, span = (uint32_t)kBins - lo;
    extern __shared__ __align__(128) uint8_t smem_ring[];
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const TopRing ring = warp_ring<TopRing>(smem_ring);
    const int64_t nrg = (p.rows + kTopRows - 1) / kTopRows;
    const int64_t n_tiles = p.ncb * nrg;
    const int64_t dcb = n_warps % p.ncb, drg = n_warps / p.ncb;
    const int64_t row_bytes = 2 * p.cols;
    TileCursor ci{warp % p.ncb, warp / p.ncb}, cb{warp % p.ncb, warp / p.ncb};
    uint32_t cmw[4] = {0u, 0u, 0u, 0u};
    int64_t cur = -1;
    auto flush_cols = [&]() {
        const int64_t c0 = cur * 256 + 8 * lane;
        if (cur >= 0 && p.colmax && c0 < p.cols) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t c = ((j & 1) ? cmw[j >> 1] >> 16 : cmw[j >> 1]) & 0x7fffu;
                if (c) atomicMax(p.colmax + c0 + j, c << 16);        // |x| as fp32 bits
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) cmw[k] = 0u;
    };
    stream_tiles_with<TopRing::NSTAGE>(
        n_tiles, warp, n_warps,
        [&](int64_t, int s) {
            const int64_t col = ci.cb * 256 + 8 * lane, r0 = ci.rg * kTopRows;
            const uint32_t d = ring.base + (uint32_t)(s * TopRing::TILE_BYTES) + ring.wr[0];
#pragma unroll
            for (int h = 0; h < kTopRows; ++h) {
                const bool ok = col < p.cols && r0 + h < p.rows;   // cols % 8 == 0: a chunk is whole or absent
                const uint8_t* src = reinterpret_cast<const uint8_t*>(p.x) + (ok ? (r0 + h) * row_bytes + 2 * col : 0);
                cp_async16(d + (uint32_t)(h * TopRing::SUB_BYTES), src, ok ? 16u : 0u);
            }
            ci.step(dcb, drg, p.ncb);
        },
        [&](int64_t, int s) {
            if (cb.cb != cur) {                                      // warp-uniform
                flush_cols();
                cur = cb.cb;
            }
            const bool col_ok = cb.cb * 256 + 8 * lane < p.cols;
            const int64_t r0 = cb.rg * kTopRows;
            uint32_t w[kTopRows][4];                                 // all four rows' reads in flight at once
#pragma unroll
            for (int h = 0; h < kTopRows; ++h) ring.read(s, h, w[h]);
#pragma unroll
            for (int h = 0; h < kTopRows; ++h)
                if (col_ok && r0 + h < p.rows) count_top(w[h], p, lo, span, cmw);
            cb.step(dcb, drg, p.ncb);
        });
    flush_cols();
}

// Histogram scans for the single-CTA kernels.  They read the 256 bucket
// totals (2 KiB), then the 128 bins of the one bucket that holds a rank or the
// maximum.
struct ScanSmem {
    unsigned long long bval[kBuckets];    // bucket totals
    unsigned long long bexcl[kBuckets];   // counts before each bucket
    unsigned long long wtot[8];           // per-warp sums of the bucket totals
    unsigned long long wexcl[8];
    unsigned long long total;
    unsigned long long need;
    int topb;                             // largest nonzero bucket, -1 if none
    int top;                              // largest nonzero bin, -1 if none
    int fb;
    int found;
};

__device__ __forceinline__ unsigned long long warp_inclusive_scan(unsigned long long v, int lane)
{
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned long long t = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += t;
    }
    return v;
}

__device__ __forceinline__ int warp_max(int v)
{
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, d));
    return v;
}

// Bucket prefix counts and the largest bin present; returns the total count.
__device__ __forceinline__ unsigned long long hist_summary(const unsigned long long* hist,
                                                           const unsigned long long* buck, ScanSmem& sm)
{
    const int t = threadIdx.x, w = t >> 5, l = t & 31;
    if (t == 0) sm.topb = -1;
    const unsigned long long v = t < kBuckets ? buck[t] : 0ull;
    const unsigned long long inc = warp_inclusive_scan(v, l);
    const int hb = warp_max(t < kBuckets && v ? t : -1);
    __syncthreads();
    if (w < kBuckets / 32 && l == 31) sm.wtot[w] = inc;
    if (l == 0 && hb >= 0) atomicMax(&sm.topb, hb);
    __syncthreads();
    if (w == 0) {
        const unsigned long long x = l < kBuckets / 32 ? sm.wtot[l] : 0ull;
        const unsigned long long iw = warp_inclusive_scan(x, l);
        if (l < kBuckets / 32) sm.wexcl[l] = iw - x;
        if (l == kBuckets / 32 - 1) sm.total = iw;
    }
    __syncthreads();
    if (t < kBuckets) {
        sm.bval[t] = v;
        sm.bexcl[t] = sm.wexcl[w] + inc - v;
    }
    if (w == 0) {                                                // largest bin of the top bucket
        int hi = -1;
        if (sm.topb >= 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (hist[128 * sm.topb + 32 * q + l]) hi = 128 * sm.topb + 32 * q + l;
        }
        hi = warp_max(hi);
        if (l == 0) sm.top = hi;
    }
    __syncthreads();
    return sm.total;
}

// The bin holding the rank-th smallest counted magnitude, 1 <= rank <= total
// (every thread gets it; hist_summary must have filled sm).
__device__ __forceinline__ int bin_at_rank(const unsigned long long* hist, unsigned long long rank, ScanSmem& sm)
{
    const int t = threadIdx.x, l = t & 31;
    if (t == 0) {                                                // in-range defaults: a rank outside
        sm.found = -1;                                           // [1, total] cannot index past the
        sm.fb = 0;                                               // histogram
        sm.need = 1;
    }
    __syncthreads();
    if (t < kBuckets) {
        const unsigned long long ex = sm.bexcl[t];
        if (rank > ex && rank <= ex + sm.bval[t]) {             // exactly one bucket
            sm.fb = t;
            sm.need = rank - ex;
        }
    }
    __syncthreads();
    if (t < 32) {
        // lane l: bins 4 l .. 4 l + 3 of the bucket, in order
        const unsigned long long* hb = hist + 128 * sm.fb + 4 * l;
        unsigned long long c[4], s = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            c[q] = hb[q];
            s += c[q];
        }
        const unsigned long long need = sm.need;
        const unsigned long long inc = warp_inclusive_scan(s, l);
        const int lane = __ffs(__ballot_sync(0xffffffffu, inc >= need)) - 1;
        if (l == lane) {
            unsigned long long run = inc - s;
            int q = 0;
            while (q < 3 && run + c[q] < need) run += c[q++];
            sm.found = 128 * sm.fb + 4 * l + q;
        }
    }
    __syncthreads();
    return sm.found;
}

struct ThresholdParams {
    const unsigned long long* shist;   // histogram of the sampled rows
    const unsigned long long* sbuck;   // its bucket totals
    double p;
    StatsCtl* ctl;
};

// L = the sampled magnitude at fraction p_low = 1 - 2(1 - p) - 8 sd of the
// sample, sd = sqrt(p (1 - p) / n_s) (0 when p_low * n_s < 1).
__global__ void __launch_bounds__(kStatThreads) outlier_threshold_kernel(ThresholdParams q)
{
    pdl_wait();
    pdl_release();
    __shared__ ScanSmem sm;
    const unsigned long long ns = hist_summary(q.shist, q.sbuck, sm);
    double plow = 1.0 - 2.0 * (1.0 - q.p) - 8.0 * sqrt(q.p * (1.0 - q.p) / (double)(ns > 0 ? ns : 1));
    if (plow < 0.0) plow = 0.0;
    const unsigned long long rank = (unsigned long long)floor(plow * (double)ns);
    const int L = rank >= 1 ? bin_at_rank(q.shist, rank, sm) : 0;
    // sample magnitudes below L: the buckets before L's, then L's bucket up to L
    if (threadIdx.x < 32) {
        const int l = threadIdx.x;
        unsigned long long below = 0;
        if (L > 0) {
            const int b0 = L & ~127;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int bin = b0 + 4 * l + k;
                if (bin < L) below += q.shist[bin];
            }
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) below += __shfl_xor_sync(0xffffffffu, below, d);
        if (l == 0) {
            if (L > 0) below += sm.bexcl[L >> 7];
            const unsigned long long at_or_above = ns - below;
            q.ctl->L = (uint32_t)(L > 0 ? L : 0);
            q.ctl->fallback = 0u;
            q.ctl->dense = (L <= 0 || at_or_above * kSparseDiv > ns) ? 1u : 0u;
        }
    }
}

struct FinalizeParams {
    const unsigned long long* hist;
    const unsigned long long* buck;
    int64_t n;
    double p;
    float* stats;
    StatsCtl* ctl;     // nullptr: hist is complete (direct path)
    int phase;         // 0: hist holds the magnitudes >= L; 1: hist is complete (gated on the fallback flag)
};

// stats[0] = the largest magnitude present, stats[1] = the magnitude of rank
// k = ceil(p n) (clamped to [1, n]).
__global__ void __launch_bounds__(kStatThreads) outlier_finalize_kernel(FinalizeParams q)
{
    pdl_wait();
    pdl_release();
    if (q.phase == 1 && q.ctl && !q.ctl->fallback) return;
    __shared__ ScanSmem sm;
    const unsigned long long counted = hist_summary(q.hist, q.buck, sm);
    long long k = (long long)ceil(q.p * (double)q.n);
    if (k < 1) k = 1;
    if (k > q.n) k = q.n;
    const unsigned long long below = (unsigned long long)q.n - counted;   // magnitudes not counted (< L)
    if (q.phase == 0 && (unsigned long long)k <= below) {
        if (threadIdx.x == 0) q.ctl->fallback = 1u;      // the rank lies below L: count those too
        return;
    }
    const int b = bin_at_rank(q.hist, (unsigned long long)k - below, sm);
    if (threadIdx.x == 0) {
        if (b >= 0) q.stats[1] = __uint_as_float((uint32_t)b << 16);
        q.stats[0] = sm.top >= 0 ? __uint_as_float((uint32_t)sm.top << 16) : 0.0f;
    }
}

// The sparse pass's grid: the resident CTAs, rounded down to a multiple that
// makes the warp count a multiple of the column blocks when that keeps at least
// half of them (each warp then keeps one column block).
cudaError_t launch_top(const uint16_t* x, int64_t rows, int64_t cols, unsigned long long* hist,
                       unsigned int* colmax, const StatsCtl* ctl, cudaStream_t s)
{
    TopParams tp{};
    tp.x = x;
    tp.rows = rows;
    tp.cols = cols;
    tp.ncb = (cols + 255) / 256;
    tp.hist = hist;
    tp.colmax = colmax;
    tp.ctl = ctl;
    const int64_t tiles = tp.ncb * ((rows + kTopRows - 1) / kTopRows);
    int grid = grid_for((const void*)outlier_top_kernel, kRingBytesPerCta, (tiles + kWarps - 1) / kWarps);
    // CTAs per whole number of column blocks: ncb / gcd(ncb, kWarps)
    int64_t a = tp.ncb, b = kWarps;
    while (b) {
        const int64_t t = a % b;
        a = b;
        b = t;
    }
    const int64_t unit = tp.ncb / a;
    if (unit <= grid && (grid / unit) * unit * 2 >= grid) grid = (int)((grid / unit) * unit);
    return launch_pdl(outlier_top_kernel, grid, kThreads, kRingBytesPerCta, s, tp);
}

int hist_grid(StatsParams& prm, int sms)
{
    const int64_t target = (int64_t)(sms > 0 ? sms : 1) * kStatThreads;
    int64_t r = target / prm.g;
    if (r < 1) r = 1;
    if (r > prm.rows) r = prm.rows;
    prm.r = r;
    prm.T = prm.g * r;
    const int64_t blocks = (prm.T + kStatThreads - 1) / kStatThreads;
    return blocks > 0x7fffffff ? -1 : (int)blocks;
}

}  // namespace

cudaError_t launch_outlier_stats(const uint16_t* x, int64_t rows, int64_t cols, double p, float* stats,
                                 float* col_absmax, void* workspace, cudaStream_t s)
{
    auto* hist = static_cast<unsigned long long*>(workspace);
    auto* shist = hist + kBins;
    auto* hbuck = shist + kBins;
    auto* sbuck = hbuck + kBuckets;
    auto* ctl = reinterpret_cast<StatsCtl*>(sbuck + kBuckets);
    cudaError_t e = cudaMemsetAsync(hist, 0, sizeof(unsigned long long) * (2 * kBins + 2 * kBuckets) + sizeof(StatsCtl), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(stats, 0, 2 * sizeof(float), s);
    if (e == cudaSuccess && col_absmax) e = cudaMemsetAsync(col_absmax, 0, sizeof(float) * (size_t)cols, s);
    if (e != cudaSuccess) return e;
    const int64_t n = rows * cols;
    if (n == 0) return cudaSuccess;

    static bool opted[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !opted[dev]) {
        e = cudaFuncSetAttribute(outlier_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kHistSmem);
        if (e != cudaSuccess) return e;
        opted[dev] = true;
    }
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

    StatsParams main{};
    main.x = x;
    main.rows = rows;
    main.row_step = 1;
    main.g = cols / 8;
    main.hist = hist;
    main.buck = hbuck;
    main.colmax = reinterpret_cast<unsigned int*>(col_absmax);
    main.ctl = ctl;
    const int main_blocks = hist_grid(main, sms);
    if (main_blocks < 0) return cudaErrorInvalidValue;

    if (n < kDirectElems) {                                   // one full histogram pass
        main.mode = kAllBins;
        outlier_hist_kernel<<<main_blocks, kStatThreads, kHistSmem, s>>>(main);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        return launch_pdl(outlier_finalize_kernel, 1, kStatThreads, 0, s, FinalizeParams{hist, hbuck, n, p, stats, nullptr, 1});
    }

    // 1. sample every s-th row (at least kSampleElems elements) and set L
    int64_t stride = n / kSampleElems;
    if (stride > kMaxSampleStride) stride = kMaxSampleStride;
    if (stride > rows) stride = rows;
    if (stride < 1) stride = 1;
    StatsParams smp = main;
    smp.rows = (rows + stride - 1) / stride;
    smp.row_step = stride;
    smp.hist = shist;
    smp.buck = sbuck;
    smp.colmax = nullptr;
    smp.mode = kAllBins;
    const int smp_blocks = hist_grid(smp, sms);
    outlier_hist_kernel<<<smp_blocks, kStatThreads, kHistSmem, s>>>(smp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_pdl(outlier_threshold_kernel, 1, kStatThreads, 0, s, ThresholdParams{shist, sbuck, p, ctl})) !=
        cudaSuccess)
        return e;
    // 2. magnitudes >= L, every channel maximum: the sparse streaming pass, or (gated on the
    //    dense flag) the shared-histogram pass
    if ((e = launch_top(x, rows, cols, hist, reinterpret_cast<unsigned int*>(col_absmax), ctl, s)) !=
        cudaSuccess)
        return e;
    main.mode = kFromLIfDense;
    if ((e = launch_pdl(outlier_hist_kernel, main_blocks, kStatThreads, kHistSmem, s, main)) != cudaSuccess)
        return e;
    if ((e = launch_pdl(outlier_finalize_kernel, 1, kStatThreads, 0, s, FinalizeParams{hist, hbuck, n, p, stats, ctl, 0})) !=
        cudaSuccess)
        return e;
    // 3. only if the rank lay below L: the rest of the histogram, and the scan again
    StatsParams rest = main;
    rest.colmax = nullptr;
    rest.mode = kBelowLIfNeeded;
    if ((e = launch_pdl(outlier_hist_kernel, main_blocks, kStatThreads, kHistSmem, s, rest)) != cudaSuccess)
        return e;
    return launch_pdl(outlier_finalize_kernel, 1, kStatThreads, 0, s, FinalizeParams{hist, hbuck, n, p, stats, ctl, 1});
}

}  // namespace fp4q
