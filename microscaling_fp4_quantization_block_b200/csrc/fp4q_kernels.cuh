// fp4q_kernels.cuh -- the streaming kernels of the FP4 block quantizer.
//
// Every kernel treats the [rows][cols] tensor as one flat run of n elements:
// blocks (block | cols) and rotation runs (rot | cols) never cross a row, so a
// block is simply `block` consecutive elements of the flat run.  A thread owns
// "units" of EPT consecutive elements (EPT = 16 or 32: one or two 256-bit
// loads), the 32 lanes of a warp own 32 consecutive units, and a warp keeps
// UNITS units per lane in flight (128 bytes of bf16 per lane) before it
// computes, walking the tensor in a grid-stride loop whose trip count is the
// same for every lane (lanes past the end hold zeros), so shuffles always see
// the full warp.  A block wider than a unit spans B/EPT adjacent lanes, whose
// maximum is combined with shuffles; a rotation run wider than a unit is
// finished with butterfly stages across K/EPT adjacent lanes.
#pragma once

#include <cuda_bf16.h>

#include "fp4q_device.cuh"

namespace fp4q {

constexpr int kThreads = 256;

template <int B, int K>
struct UnitShape {
    static constexpr int kMaxBK = (B > K ? B : K);
    static constexpr int EPT = kMaxBK <= 16 ? 16 : 32;           // elements per unit
    static constexpr int UNITS = EPT == 16 ? 4 : 2;              // units in flight per lane
    static constexpr int kBlocksPerUnit = B <= EPT ? EPT / B : 1;
    static constexpr int kLanesPerBlock = B <= EPT ? 1 : B / EPT;
    static constexpr int kChunk = K == 0 ? 1 : (K <= EPT ? K : EPT); // in-register run
    static constexpr int kRotLanes = K > EPT ? K / EPT : 1;
    static constexpr int kBlockElems = B <= EPT ? B : EPT;        // elements of a block in one unit
    static_assert(kLanesPerBlock <= 32 && kRotLanes <= 32, "block or rotation wider than a warp");
};

// ---------------------------------------------------------------- unit loads
// Raw bf16 words of one unit (word k = elements 2k, 2k+1).  A unit that runs
// past n (only the last one) is read element by element and zero-padded; the
// padding occupies whole blocks and rotation runs because n is a multiple of
// both, so it never mixes with real data.
template <int EPT>
__device__ __forceinline__ void load_unit(const uint16_t* __restrict__ x, int64_t n, int64_t u,
                                          uint32_t (&w)[EPT / 2])
{
    const int64_t e0 = u * EPT;
    if (e0 + EPT <= n) {
#pragma unroll
        for (int h = 0; h < EPT / 16; ++h) {
            U32x8 r = ldg256_stream(x + e0 + 16 * h);
#pragma unroll
            for (int k = 0; k < 8; ++k) w[8 * h + k] = r.v[k];
        }
    } else {
#pragma unroll
        for (int k = 0; k < EPT / 2; ++k) {
            uint32_t lo = (e0 + 2 * k < n) ? (uint32_t)x[e0 + 2 * k] : 0u;
            uint32_t hi = (e0 + 2 * k + 1 < n) ? (uint32_t)x[e0 + 2 * k + 1] : 0u;
            w[k] = lo | (hi << 16);
        }
    }
}

template <int EPT>
__device__ __forceinline__ void unpack_unit(const uint32_t (&w)[EPT / 2], float (&v)[EPT])
{
#pragma unroll
    for (int k = 0; k < EPT / 2; ++k) {
        v[2 * k] = bf16_lo(w[k]);
        v[2 * k + 1] = bf16_hi(w[k]);
    }
}

// Optional rotation of a unit held in registers: runs of K elements, the part
// inside the unit in registers, the rest across lanes, then 1/sqrt(K).
template <int B, int K>
__device__ __forceinline__ void rotate_unit(float (&v)[UnitShape<B, K>::EPT], int lane, float c_hi,
                                            float c_lo)
{
    using S = UnitShape<B, K>;
    if constexpr (K > 0) {
        fwht_inreg<S::EPT, S::kChunk>(v);
        if constexpr (S::kRotLanes > 1) fwht_xlane<S::EPT, S::kRotLanes>(v, lane);
        normalize<S::EPT>(v, c_hi, c_lo);
    }
}

// Per-block absolute maximum of a unit (combined across lanes for wide blocks).
template <int B, int K>
__device__ __forceinline__ void block_max(const float (&v)[UnitShape<B, K>::EPT],
                                          float (&m)[UnitShape<B, K>::kBlocksPerUnit])
{
    using S = UnitShape<B, K>;
#pragma unroll
    for (int bi = 0; bi < S::kBlocksPerUnit; ++bi) {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < S::kBlockElems; ++i) a = fmaxf(a, fabsf(v[bi * S::kBlockElems + i]));
        m[bi] = a;
    }
    if constexpr (S::kLanesPerBlock > 1) m[0] = group_max<S::kLanesPerBlock>(m[0]);
}

// ---------------------------------------------------------------- quantize
struct QuantParams {
    const uint16_t* x;     // bf16 bits
    int64_t n;             // elements
    uint8_t* codes;        // n/2 bytes
    uint8_t* scales;       // n/B bytes
    const float* gsrc;     // per-tensor scale G (nullptr: G = 1)
    float c_hi, c_lo;      // 1/sqrt(K) split in two fp32 parts
};

template <int FMT, int B, int K>
__device__ __forceinline__ void quantize_unit(const QuantParams& p, int64_t u, const uint32_t (&w)[UnitShape<B, K>::EPT / 2],
                                              int lane, float G, float denom)
{
    using S = UnitShape<B, K>;
    constexpr int EPT = S::EPT;
    constexpr int NB = S::kBlocksPerUnit;
    float v[EPT];
    unpack_unit<EPT>(w, v);
    rotate_unit<B, K>(v, lane, p.c_hi, p.c_lo);

    float m[NB];
    block_max<B, K>(v, m);

    float sc[NB], rc[NB];
    uint32_t code[NB];
    bool slow_scale = false;
#pragma unroll
    for (int bi = 0; bi < NB; ++bi) {
        code[bi] = block_scale<FMT>(m[bi], G, denom, sc[bi], rc[bi]);
        if constexpr (FMT != kE8M0) {
            if (sc[bi] == 0.0f) rc[bi] = 0.0f;                       // zero-rounded block
            else if (!scale_product_safe(sc[bi])) slow_scale = true;
        }
    }

    uint32_t cw[EPT / 8];
    if constexpr (FMT == kE8M0) {
        // S is a power of two: y * (1/S) is exact, so it is the quotient itself.
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k) {
            float q[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = 8 * k + j;
                q[j] = __fmul_rn(v[i], rc[i / S::kBlockElems]);
            }
            cw[k] = e2m1_pack8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
        }
    } else {
        bool agree = !slow_scale;
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k) {
            float lo[8], hi[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = 8 * k + j;
                const float q0 = __fmul_rn(v[i], rc[i / S::kBlockElems]);
                lo[j] = __fmul_rn(q0, kBracketLo);
                hi[j] = __fmul_rn(q0, kBracketHi);
            }
            const uint32_t a = e2m1_pack8(lo[0], lo[1], lo[2], lo[3], lo[4], lo[5], lo[6], lo[7]);
            const uint32_t b = e2m1_pack8(hi[0], hi[1], hi[2], hi[3], hi[4], hi[5], hi[6], hi[7]);
            agree = agree && (a == b);
            cw[k] = a;
        }
        if (!agree) {
            // rare: a quotient near an E2M1 rounding threshold, or an extreme scale
#pragma unroll
            for (int k = 0; k < EPT / 8; ++k) {
                float q[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = 8 * k + j;
                    const float s = sc[i / S::kBlockElems];
                    q[j] = s != 0.0f ? __fdiv_rn(v[i], s) : 0.0f;
                }
                cw[k] = e2m1_pack8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
            }
        }
        // zero-rounded blocks store plain 0x0 nibbles
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k)
            if (sc[(8 * k) / S::kBlockElems] == 0.0f) cw[k] = 0u;
    }

    // ---- stores
    const int64_t e0 = u * EPT;
    if (e0 >= p.n) return;
    uint8_t* cdst = p.codes + e0 / 2;
    if (e0 + EPT <= p.n) {
        if constexpr (EPT == 16) stg64(cdst, cw[0], cw[1]);
        else stg128(cdst, cw[0], cw[1], cw[2], cw[3]);
    } else {
        const int nbytes = (int)((p.n - e0) / 2);
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (4 * k + j < nbytes) cdst[4 * k + j] = (uint8_t)(cw[k] >> (8 * j));
    }
    if constexpr (S::kLanesPerBlock > 1) {
        if ((lane % S::kLanesPerBlock) == 0) p.scales[e0 / B] = (uint8_t)code[0];
    } else {
        const int64_t b0 = e0 / B;
        const int64_t nblk = p.n / B;
        if (e0 + EPT <= p.n) {
            if constexpr (NB == 1) {
                p.scales[b0] = (uint8_t)code[0];
            } else if constexpr (NB == 2) {
                *reinterpret_cast<uint16_t*>(p.scales + b0) = (uint16_t)(code[0] | (code[1] << 8));
            } else if constexpr (NB == 4) {
                *reinterpret_cast<uint32_t*>(p.scales + b0) =
                    code[0] | (code[1] << 8) | (code[2] << 16) | (code[3] << 24);
            } else {
#pragma unroll
                for (int bi = 0; bi < NB; ++bi) p.scales[b0 + bi] = (uint8_t)code[bi];
            }
        } else {
#pragma unroll
            for (int bi = 0; bi < NB; ++bi)
                if (b0 + bi < nblk) p.scales[b0 + bi] = (uint8_t)code[bi];
        }
    }
}

template <int FMT, int B, int K>
__global__ void __launch_bounds__(kThreads) quantize_kernel(QuantParams p)
{
    using S = UnitShape<B, K>;
    constexpr int EPT = S::EPT, U = S::UNITS;
    const int lane = threadIdx.x & 31;
    const int64_t n_units = (p.n + EPT - 1) / EPT;
    const int64_t n_tiles = (n_units + 32 * U - 1) / (32 * U);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;

    float G = 1.0f;
    if (FMT != kE8M0 && p.gsrc != nullptr) G = *p.gsrc;
    const float denom = __fmul_rn(6.0f, G);

    for (int64_t tile = warp; tile < n_tiles; tile += n_warps) {
        uint32_t w[U][EPT / 2];
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t u = (tile * U + j) * 32 + lane;
            load_unit<EPT>(p.x, p.n, u, w[j]);
        }
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t u = (tile * U + j) * 32 + lane;
            quantize_unit<FMT, B, K>(p, u, w[j], lane, G, denom);
        }
    }
}

// ---------------------------------------------------------------- per-tensor amax
struct AmaxParams {
    const uint16_t* x;
    int64_t n;
    unsigned int* amax_bits;   // max |y| as fp32 bits (non-negative floats order as integers)
    float c_hi, c_lo;
};

template <int K>
__global__ void __launch_bounds__(kThreads) amax_kernel(AmaxParams p)
{
    using S = UnitShape<16, K>;
    constexpr int EPT = S::EPT, U = S::UNITS;
    const int lane = threadIdx.x & 31;
    const int64_t n_units = (p.n + EPT - 1) / EPT;
    const int64_t n_tiles = (n_units + 32 * U - 1) / (32 * U);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    float mx = 0.0f;
    for (int64_t tile = warp; tile < n_tiles; tile += n_warps) {
        uint32_t w[U][EPT / 2];
#pragma unroll
        for (int j = 0; j < U; ++j) load_unit<EPT>(p.x, p.n, (tile * U + j) * 32 + lane, w[j]);
#pragma unroll
        for (int j = 0; j < U; ++j) {
            float v[EPT];
            unpack_unit<EPT>(w[j], v);
            rotate_unit<16, K>(v, lane, p.c_hi, p.c_lo);
#pragma unroll
            for (int i = 0; i < EPT; ++i) mx = fmaxf(mx, fabsf(v[i]));
        }
    }
    mx = group_max<32>(mx);
    if (lane == 0 && mx > 0.0f) atomicMax(p.amax_bits, __float_as_uint(mx));
}

// G = amax / (6 * 448) (correctly rounded), or 1 for an all-zero tensor.
static __global__ void global_scale_kernel(const float* amax_in, float* gscale)
{
    const float amax = *amax_in;
    *gscale = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// ---------------------------------------------------------------- codes / scales of a unit
template <int EPT>
__device__ __forceinline__ void load_codes(const uint8_t* __restrict__ codes, int64_t n, int64_t u,
                                           uint32_t (&cw)[EPT / 8])
{
    const int64_t e0 = u * EPT;
    const uint8_t* src = codes + e0 / 2;
    if (e0 + EPT <= n) {
        if constexpr (EPT == 16) {
            uint2 r = __ldg(reinterpret_cast<const uint2*>(src));
            cw[0] = r.x;
            cw[1] = r.y;
        } else {
            uint4 r = __ldg(reinterpret_cast<const uint4*>(src));
            cw[0] = r.x;
            cw[1] = r.y;
            cw[2] = r.z;
            cw[3] = r.w;
        }
    } else {
        const int64_t nbytes = e0 < n ? (n - e0) / 2 : 0;
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (4 * k + j < nbytes) word |= (uint32_t)src[4 * k + j] << (8 * j);
            cw[k] = word;
        }
    }
}

// Block scales S of a unit (decoded; G applied for the UE formats).
template <int B, int K>
__device__ __forceinline__ void load_scales(const uint8_t* __restrict__ scales, int fmt, float G,
                                            int64_t n, int64_t u,
                                            float (&S)[UnitShape<B, K>::kBlocksPerUnit])
{
    using Sh = UnitShape<B, K>;
    const int64_t e0 = u * Sh::EPT;
#pragma unroll
    for (int bi = 0; bi < Sh::kBlocksPerUnit; ++bi) {
        const int64_t e = e0 + (int64_t)bi * Sh::kBlockElems;
        uint32_t c = e < n ? (uint32_t)__ldg(scales + e / B) : 0u;
        float s;
        if (fmt == kE8M0) s = e < n ? e8m0_decode(c) : 0.0f;
        else if (fmt == kUE4M3) s = __fmul_rn(ue4m3_decode(c), G);
        else s = __fmul_rn(ue5m3_decode(c), G);
        S[bi] = s;
    }
}

// Dequantized values of a unit: v = fp32(decode(nibble) * S).
template <int B, int K>
__device__ __forceinline__ void decode_unit(const uint32_t (&cw)[UnitShape<B, K>::EPT / 8],
                                            const float (&S)[UnitShape<B, K>::kBlocksPerUnit],
                                            float (&v)[UnitShape<B, K>::EPT])
{
    using Sh = UnitShape<B, K>;
#pragma unroll
    for (int k = 0; k < Sh::EPT / 8; ++k) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = 8 * k + 2 * j;
            float lo, hi;
            e2m1_unpack2((cw[k] >> (8 * j)) & 0xffu, lo, hi);
            const float s = S[i / Sh::kBlockElems];
            v[i] = __fmul_rn(lo, s);
            v[i + 1] = __fmul_rn(hi, s);
        }
    }
}

// ---------------------------------------------------------------- dequantize
struct DequantParams {
    const uint8_t* codes;
    const uint8_t* scales;
    const float* gsrc;     // nullptr: G = 1
    int64_t n;
    int fmt;
    void* y;               // bf16 or fp32 output
    float c_hi, c_lo;
};

template <int B, int K, bool F32OUT>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(DequantParams p)
{
    using S = UnitShape<B, K>;
    constexpr int EPT = S::EPT, U = S::UNITS;
    const int lane = threadIdx.x & 31;
    const int64_t n_units = (p.n + EPT - 1) / EPT;
    const int64_t n_tiles = (n_units + 32 * U - 1) / (32 * U);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const float G = (p.fmt != kE8M0 && p.gsrc != nullptr) ? *p.gsrc : 1.0f;

    for (int64_t tile = warp; tile < n_tiles; tile += n_warps) {
        uint32_t cw[U][EPT / 8];
        float sc[U][S::kBlocksPerUnit];
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t u = (tile * U + j) * 32 + lane;
            load_codes<EPT>(p.codes, p.n, u, cw[j]);
            load_scales<B, K>(p.scales, p.fmt, G, p.n, u, sc[j]);
        }
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t u = (tile * U + j) * 32 + lane;
            float v[EPT];
            decode_unit<B, K>(cw[j], sc[j], v);
            rotate_unit<B, K>(v, lane, p.c_hi, p.c_lo);
            const int64_t e0 = u * EPT;
            if (e0 >= p.n) continue;
            const bool full = e0 + EPT <= p.n;
            if constexpr (F32OUT) {
                float* dst = reinterpret_cast<float*>(p.y) + e0;
                if (full) {
#pragma unroll
                    for (int k = 0; k < EPT / 4; ++k)
                        stg128(dst + 4 * k, __float_as_uint(v[4 * k]), __float_as_uint(v[4 * k + 1]),
                               __float_as_uint(v[4 * k + 2]), __float_as_uint(v[4 * k + 3]));
                } else {
                    for (int i = 0; i < EPT && e0 + i < p.n; ++i) dst[i] = v[i];
                }
            } else {
                uint32_t o[EPT / 2];
#pragma unroll
                for (int k = 0; k < EPT / 2; ++k) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
                    o[k] = *reinterpret_cast<uint32_t*>(&h);
                }
                uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(p.y) + e0);
                if (full) {
#pragma unroll
                    for (int k = 0; k < EPT / 8; ++k) stg128(dst + 4 * k, o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
                } else {
                    for (int k = 0; k < EPT / 2 && e0 + 2 * k < p.n; ++k) dst[k] = o[k];
                }
            }
        }
    }
}

// ---------------------------------------------------------------- block MSE
struct MseParams {
    const uint16_t* x;
    const uint8_t* codes;
    const uint8_t* scales;
    const float* gsrc;
    int64_t n;
    int fmt;
    float* block_mse;      // n/B floats or nullptr
    double* partials;      // [gridDim.x][4]
    float c_hi, c_lo;
};

template <int N>
__device__ __forceinline__ float tree_sum(const float* a)
{
    if constexpr (N == 1) return a[0];
    else return __fadd_rn(tree_sum<N / 2>(a), tree_sum<N / 2>(a + N / 2));
}

template <int LANES>
__device__ __forceinline__ float group_sum(float s)
{
#pragma unroll
    for (int d = 1; d < LANES; d <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, d));
    return s;
}

template <int B, int K>
__global__ void __launch_bounds__(kThreads) block_mse_kernel(MseParams p)
{
    using S = UnitShape<B, K>;
    constexpr int EPT = S::EPT, U = S::UNITS, NB = S::kBlocksPerUnit, BE = S::kBlockElems;
    constexpr int LPB = S::kLanesPerBlock;
    const int lane = threadIdx.x & 31;
    const int64_t n_units = (p.n + EPT - 1) / EPT;
    const int64_t n_tiles = (n_units + 32 * U - 1) / (32 * U);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const float G = (p.fmt != kE8M0 && p.gsrc != nullptr) ? *p.gsrc : 1.0f;

    double acc_total = 0.0, acc_nonmax = 0.0, acc_max = 0.0, acc_zero = 0.0;
    for (int64_t tile = warp; tile < n_tiles; tile += n_warps) {
        uint32_t w[U][EPT / 2];
        uint32_t cw[U][EPT / 8];
        float sc[U][NB];
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t u = (tile * U + j) * 32 + lane;
            load_unit<EPT>(p.x, p.n, u, w[j]);
            load_codes<EPT>(p.codes, p.n, u, cw[j]);
            load_scales<B, K>(p.scales, p.fmt, G, p.n, u, sc[j]);
        }
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int64_t u = (tile * U + j) * 32 + lane;
            const int64_t e0 = u * EPT;
            float y[EPT], v[EPT];
            unpack_unit<EPT>(w[j], y);
            rotate_unit<B, K>(y, lane, p.c_hi, p.c_lo);
            decode_unit<B, K>(cw[j], sc[j], v);
            float m[NB];
            block_max<B, K>(y, m);
#pragma unroll
            for (int bi = 0; bi < NB; ++bi) {
                float e2[BE];
                float vmax = 0.0f;
                int first = BE;                       // first element of largest |y| in this lane
#pragma unroll
                for (int i = BE - 1; i >= 0; --i) {
                    const float yi = y[bi * BE + i], vi = v[bi * BE + i];
                    const float d = __fsub_rn(yi, vi);
                    e2[i] = __fmul_rn(d, d);
                    vmax = fmaxf(vmax, fabsf(vi));
                    if (fabsf(yi) == m[bi]) first = i;
                }
                float emax = 0.0f;
#pragma unroll
                for (int i = 0; i < BE; ++i) if (i == first) emax = e2[i];
                bool owner = first < BE;
                if constexpr (LPB > 1) {
                    // the block's maximum belongs to the lowest lane that holds it
                    const unsigned grp = (lane / LPB) * LPB;
                    const unsigned mask = ((LPB == 32) ? 0xffffffffu : ((1u << LPB) - 1u)) << grp;
                    const unsigned holders = __ballot_sync(0xffffffffu, owner) & mask;
                    owner = owner && (__ffs(holders) - 1 == lane);
                    vmax = group_max<LPB>(vmax);
                }
                const float sum = tree_sum<BE>(e2);
                const float mx = owner ? emax : 0.0f;
                // non-max part: every element except the owner's first maximum
                float nm_arr[BE];
#pragma unroll
                for (int i = 0; i < BE; ++i) nm_arr[i] = (owner && i == first) ? 0.0f : e2[i];
                float nonmax = tree_sum<BE>(nm_arr);
                float bsum = sum, bmax = mx;
                if constexpr (LPB > 1) {
                    bsum = group_sum<LPB>(bsum);
                    nonmax = group_sum<LPB>(nonmax);
                    bmax = group_sum<LPB>(bmax);
                }
                const int64_t eb = e0 + (int64_t)bi * BE;
                const bool leader = (LPB == 1) || ((lane % LPB) == 0);
                if (leader && eb < p.n) {
                    if (p.block_mse) p.block_mse[eb / B] = __fdiv_rn(bsum, (float)B);
                    acc_total += (double)bsum;
                    if (vmax == 0.0f) acc_zero += (double)bsum;
                    else {
                        acc_nonmax += (double)nonmax;
                        acc_max += (double)bmax;
                    }
                }
            }
        }
    }
    // deterministic block reduction: warp butterflies, then warps in order
    __shared__ double red[kThreads / 32][4];
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
        acc_total += __shfl_xor_sync(0xffffffffu, acc_total, d);
        acc_nonmax += __shfl_xor_sync(0xffffffffu, acc_nonmax, d);
        acc_max += __shfl_xor_sync(0xffffffffu, acc_max, d);
        acc_zero += __shfl_xor_sync(0xffffffffu, acc_zero, d);
    }
    const int wid = threadIdx.x >> 5;
    if (lane == 0) {
        red[wid][0] = acc_total;
        red[wid][1] = acc_nonmax;
        red[wid][2] = acc_max;
        red[wid][3] = acc_zero;
    }
    __syncthreads();
    if (threadIdx.x < 4) {
        double s = 0.0;
        for (int k = 0; k < kThreads / 32; ++k) s += red[k][threadIdx.x];
        p.partials[(int64_t)blockIdx.x * 4 + threadIdx.x] = s;
    }
}

// terms[i] = (sum of partials[*][i]) / n, summed in a fixed order.
static __global__ void __launch_bounds__(kThreads) mse_finalize_kernel(const double* partials, int nparts,
                                                               int64_t n, double* terms)
{
    __shared__ double red[kThreads][4];
    double s[4] = {0.0, 0.0, 0.0, 0.0};
    for (int i = threadIdx.x; i < nparts; i += kThreads)
#pragma unroll
        for (int k = 0; k < 4; ++k) s[k] += partials[(int64_t)i * 4 + k];
#pragma unroll
    for (int k = 0; k < 4; ++k) red[threadIdx.x][k] = s[k];
    __syncthreads();
    for (int h = kThreads / 2; h >= 1; h >>= 1) {
        if (threadIdx.x < h)
#pragma unroll
            for (int k = 0; k < 4; ++k) red[threadIdx.x][k] += red[threadIdx.x + h][k];
        __syncthreads();
    }
    if (threadIdx.x < 4) terms[threadIdx.x] = n > 0 ? red[0][threadIdx.x] / (double)n : 0.0;
}

// ---------------------------------------------------------------- element codecs
static __global__ void __launch_bounds__(kThreads) e2m1_encode_kernel(const float* __restrict__ r, int64_t n,
                                                              uint8_t* __restrict__ out)
{
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; 8 * i < n; i += stride) {
        const int64_t e = 8 * i;
        float q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = (e + j < n) ? r[e + j] : 0.0f;
        const uint32_t w = e2m1_pack8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
        if (e + 8 <= n) {
            *reinterpret_cast<uint32_t*>(out + e / 2) = w;
        } else {
            for (int j = 0; 2 * j < n - e; ++j) out[e / 2 + j] = (uint8_t)(w >> (8 * j));
        }
    }
}

static __global__ void __launch_bounds__(kThreads) scale_encode_kernel(const float* __restrict__ s, int64_t n,
                                                               int fmt, uint8_t* __restrict__ out)
{
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
        const float v = s[i];
        uint32_t c;
        if (fmt == kE8M0) c = e8m0_from_amax(v);
        else if (fmt == kUE4M3) c = ue4m3_encode(v);
        else c = ue5m3_encode(v);
        out[i] = (uint8_t)c;
    }
}

}  // namespace fp4q
