// fp4q_gscale.cu -- MSE-optimised per-tensor scale ("Bridging the Gap", s3.2,
// MR-GPTQ item 2: the global scale is optimised together with the group
// scales instead of being set by the max rule alone).
//
// Candidates G_j = fp32(G0 (16 + j) / 16) for j in [-below, above] (from half to
// almost twice the max-rule G0 = amax / 2688, 1 for an all-zero tensor), tried
// in the order j = 0, 1, -1, 2, -2, ...; under each the block scales follow the
// max rule, and the candidate of least total squared error is kept (a strictly
// smaller error replaces the best, so G0 wins every tie).
//
// One pass over x computes the error of every candidate at once: each unit of
// 32 elements is widened (and rotated) once, its block maxima taken once, and
// then, per candidate, its scale codes, E2M1 codes, decoded values and squared
// errors are formed exactly as the quantizer forms them (fp32 per block).  A
// warp folds its lanes' unit errors in a fixed order into per-warp fp64
// accumulators in shared memory; each CTA writes one fp64 partial per
// candidate; the CTA that finishes last sums the partials in CTA order, picks
// the candidate and writes G* and the per-candidate errors (deterministic).
#include <cstring>

#include "../../include/fp4q.h"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

constexpr int kMaxCand = 24;                // 8 below + 15 above + G0

struct GscaleParams {
    const uint16_t* x;
    int64_t n;
    const float* amax;          // tensor maximum of the (rotated) tensor
    float c_hi, c_lo;
    int below, above;
    double* partials;           // [gridDim.x][kMaxCand]
    unsigned int* done;         // completion counter (0 at launch, left 0)
    float* gscale;              // out: G*
    double* errors;             // out (optional): per-candidate per-tensor MSE, index j + below
};

// Dynamic shared memory after the ring (and the rotation scratch): per-candidate
// scale tables, constants and the per-warp error accumulators.
constexpr int kTabBytes = kMaxCand * 256 * (int)sizeof(float2);
constexpr int kConstBytes = kMaxCand * (int)sizeof(float4);
constexpr int kAccBytes = kWarps * kMaxCand * (int)sizeof(double);
template <int K>
constexpr int smem_bytes()
{
    return ring_smem_bytes<K>() + kTabBytes + kConstBytes + kAccBytes;
}

// Squared error of one unit under one candidate scale: the unit's share of its
// blocks' errors (fp32 sums of fp32 terms, as the fused MSE forms them).
template <int FMT, int B, int K>
__device__ __forceinline__ float unit_error(const f32x2 (&v)[EPT / 2], const float (&m)[UnitShape<B, K>::NB],
                                            const ScaleConsts& kc, const float2* tab, float nz)
{
    using S = UnitShape<B, K>;
    constexpr int NB = S::NB, BE = S::BE;
    float sc[NB], rm[NB];
    uint32_t code[NB];
    const bool exact = unit_scales<FMT, NB>(m, kc, tab, code, sc, rm);
    const f32x2 nz2 = pk(nz, nz);
    f32x2 acc = pk(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < EPT / 8; ++k) {
        const int bi = (8 * k) / BE;
        const f32x2* vk = v + 4 * k;
        uint32_t h[4];
        if (exact) {
            const f32x2 R2 = pk(rm[bi], rm[bi]), nS2 = pk(-sc[bi], -sc[bi]);
            pack_pairs_dec(div2_cr(vk[0], R2, nS2), div2_cr(vk[1], R2, nS2), div2_cr(vk[2], R2, nS2),
                           div2_cr(vk[3], R2, nS2), h);
        } else {
            const uint32_t cw = sc[bi] != 0.0f ? pack_pairs_div(vk[0], vk[1], vk[2], vk[3], sc[bi]) : 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t hh;
                asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
                    : "=r"(hh)
                    : "r"((cw >> (8 * j)) & 0xffu));
                h[j] = hh;
            }
        }
        const f32x2 s2 = pk(sc[bi], sc[bi]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __half2 hh = *reinterpret_cast<__half2*>(&h[j]);
            const f32x2 g = pk(__low2float(hh), __high2float(hh));
            const f32x2 d = sub2(vk[j], fma2(g, s2, nz2));         // y - fp32(g S); S = 0 gives v = 0
            acc = fma2(d, d, acc);
        }
    }
    float a, b;
    upk(acc, a, b);
    return __fadd_rn(a, b);
}

template <int FMT, int B, int K>
__global__ void __launch_bounds__(kThreads, 1) gscale_search_kernel(GscaleParams p)
{
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int kTab0 = ring_smem_bytes<K>();
    float2* tabs = reinterpret_cast<float2*>(smem + kTab0);
    float4* consts = reinterpret_cast<float4*>(smem + kTab0 + kTabBytes);
    double* wacc = reinterpret_cast<double*>(smem + kTab0 + kTabBytes + kConstBytes);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nc = p.below + p.above + 1;
    const float amax = *p.amax;
    const float g0 = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    // candidate c = j + below: G_j = fp32(G0 (16 + j) / 16), (16 + j) / 16 exact
    for (int c = 0; c < nc; ++c) {
        const float G = __fmul_rn(g0, (float)(16 + c - p.below) * 0.0625f);
        fill_scale_table<FMT>(tabs + 256 * c, G);
        if (threadIdx.x == 0) {
            const ScaleConsts kc = scale_consts(G);
            consts[c] = make_float4(kc.G, kc.denom, kc.rdenom, kc.denom_ok ? 1.0f : 0.0f);
        }
    }
    for (int i = threadIdx.x; i < kWarps * kMaxCand; i += kThreads) wacc[i] = 0.0;
    __syncthreads();

    const int64_t n_tiles = (p.n + 32 * EPT - 1) / (32 * EPT);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const XRing ring = warp_ring<XRing, K>(smem);
    const float nz = __uint_as_float(0x80000000u | (uint32_t)((uint64_t)p.n >> 63));
    using S = UnitShape<B, K>;
    stream_tiles(ring, reinterpret_cast<const uint8_t*>(p.x), 2 * p.n, n_tiles, warp, n_warps, lane,
                 [&](int64_t t, int s) {
                     uint32_t w[EPT / 2];
                     ring.read(s, 0, w);
                     f32x2 v[EPT / 2];
                     load_unit<K>(w, v, lane, p.c_hi, p.c_lo);
                     float m[S::NB];
                     if constexpr (K == 0) block_max_words<B>(w, m);
                     else block_max<B, K>(v, m);
                     const bool live = (t * 32 + lane) * EPT < p.n;      // lanes past the end hold zeros
                     for (int c = 0; c < nc; ++c) {
                         const float4 k4 = consts[c];
                         ScaleConsts kc;
                         kc.G = k4.x;
                         kc.denom = k4.y;
                         kc.rdenom = k4.z;
                         kc.denom_ok = k4.w != 0.0f;
                         const float e = live ? unit_error<FMT, B, K>(v, m, kc, tabs + 256 * c, nz) : 0.0f;
                         double d = (double)e;
#pragma unroll
                         for (int o = 16; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                         if (lane == 0) wacc[wid * kMaxCand + c] += d;
                     }
                 });
    __syncthreads();
    // CTA partials (warps in index order), then the last CTA finishes
    for (int c = threadIdx.x; c < nc; c += kThreads) {
        double s = 0.0;
        for (int w = 0; w < kWarps; ++w) s += wacc[w * kMaxCand + c];
        p.partials[(int64_t)blockIdx.x * kMaxCand + c] = s;
    }
    __shared__ bool last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicInc(p.done, gridDim.x - 1u) == gridDim.x - 1u;
    __syncthreads();
    if (!last) return;
    __threadfence();
    __shared__ double tot[kMaxCand];
    for (int c = threadIdx.x; c < nc; c += kThreads) {
        double s = 0.0;
        for (int b = 0; b < (int)gridDim.x; ++b) s += __ldcg(p.partials + (int64_t)b * kMaxCand + c);
        tot[c] = s;
        if (p.errors) p.errors[c] = s / (double)p.n;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int best = 0;                                   // j = 0
        double best_err = tot[p.below];
        const int span = p.below > p.above ? p.below : p.above;
        for (int t = 1; t <= 2 * span; ++t) {
            const int j = (t & 1) ? (t + 1) / 2 : -(t / 2);
            if (j > p.above || -j > p.below) continue;
            if (tot[j + p.below] < best_err) {
                best = j;
                best_err = tot[j + p.below];
            }
        }
        *p.gscale = __fmul_rn(g0, (float)(16 + best) * 0.0625f);
    }
}

template <int FMT, int B, int K>
cudaError_t run_gscale(const GscaleParams& p, cudaStream_t s)
{
    auto kern = gscale_search_kernel<FMT, B, K>;
    int64_t need = ring_ctas_needed(p.n, EPT);
    if (need > kMaxPartialCtas) need = kMaxPartialCtas;
    const int grid = grid_for((const void*)kern, smem_bytes<K>(), need);
    kern<<<grid, kThreads, smem_bytes<K>(), s>>>(p);
    return cudaGetLastError();
}

template <int FMT, int B>
cudaError_t gscale_by_rot(int K, const GscaleParams& p, cudaStream_t s)
{
    switch (K) {
    case 0: return run_gscale<FMT, B, 0>(p, s);
    case 16: return run_gscale<FMT, B, 16>(p, s);
    case 32: return run_gscale<FMT, B, 32>(p, s);
    case 128: return run_gscale<FMT, B, 128>(p, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t gscale_by_block(int B, int K, const GscaleParams& p, cudaStream_t s)
{
    switch (B) {
    case 8: return gscale_by_rot<FMT, 8>(K, p, s);
    case 16: return gscale_by_rot<FMT, 16>(K, p, s);
    case 32: return gscale_by_rot<FMT, 32>(K, p, s);
    case 64: return gscale_by_rot<FMT, 64>(K, p, s);
    case 128: return gscale_by_rot<FMT, 128>(K, p, s);
    case 256: return gscale_by_rot<FMT, 256>(K, p, s);
    default: return cudaErrorInvalidValue;
    }
}

// Workspace: completion counter (16 B), the tensor maximum (16 B), then the
// per-CTA partials.
constexpr size_t kWsHeader = 32;

}  // namespace

cudaError_t launch_gscale_search(const uint16_t* x, int64_t n, int fmt, int block, int rot, float c_hi, float c_lo,
                                 int below, int above, float* gscale, double* errors, void* workspace, cudaStream_t s)
{
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    GscaleParams p{};
    p.x = x;
    p.n = n;
    p.amax = reinterpret_cast<const float*>(ws + 16);
    p.c_hi = c_hi;
    p.c_lo = c_lo;
    p.below = below;
    p.above = above;
    p.partials = reinterpret_cast<double*>(ws + kWsHeader);
    p.done = reinterpret_cast<unsigned int*>(ws);
    p.gscale = gscale;
    p.errors = errors;
    switch (fmt) {
    case kUE4M3: return gscale_by_block<kUE4M3>(block, rot, p, s);
    case kUE5M3: return gscale_by_block<kUE5M3>(block, rot, p, s);
    default: return cudaErrorInvalidValue;
    }
}

size_t gscale_workspace_bytes() { return kWsHeader + (size_t)kMaxPartialCtas * kMaxCand * sizeof(double); }

}  // namespace fp4q
