// fp4q_kernels.cuh -- the streaming kernels of the FP4 block quantizer.
//
// Every kernel treats the [rows][cols] tensor as one flat run of n elements:
// blocks (block | cols) and rotation runs (rot | cols) never cross a row, so a
// block is simply `block` consecutive elements of the flat run.
//
// Work decomposition.  A lane owns "units" of 32 consecutive elements; the 32
// lanes of a warp own the 32 consecutive units of a 1024-element "tile"
// (quantize, amax, MSE), so blocks of 8, 16 or 32 sit inside one lane, wider
// blocks span adjacent lanes (maxima combined with shuffles), and a 128-wide
// rotation run spans 4 lanes, which trade halves of it through shared memory
// (unit_sums).  Warps walk tiles in a grid-stride loop with the same trip
// count for every lane (lanes past the end hold zeros), so shuffles and warp
// barriers always see the whole warp.
//
// Memory pipeline.  The streamed input goes through a per-warp ring of
// NSTAGE tiles in shared memory filled with 16-byte cp.async copies: while a
// warp computes tile i, tiles i+1 .. i+NSTAGE-1 are in flight (6 KB per warp),
// independent of the compute.  Each copy instruction moves 512 contiguous
// bytes per warp; chunks land XOR-swizzled so each lane reads its own unit
// back with conflict-free 128-bit shared loads.
//
// Arithmetic.  Element values live as fp32 pairs (f32x2) so that products,
// sums and butterflies issue as packed two-wide instructions; the scales of
// two blocks are computed together the same way.  The quantizer keeps its
// work on the floating-point (FMA) pipe where it can: on sm_100 the integer /
// logic pipe that runs converts, permutes, min/max and compares issues at
// half the rate, so codes come from exactly computed quotients (div2_cr) and
// one convert per pair, bf16 is widened by a mixed-precision add, and unrotated
// block maxima use packed bf16 magnitude maxima.
#pragma once

#include <cuda_bf16.h>

#include "fp4q_device.cuh"

namespace fp4q {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRingBytesPerWarp = 8192;
constexpr int kRingBytesPerCta = kRingBytesPerWarp * kWarps;
constexpr int EPT = 32;                                          // elements per unit

template <int B, int K>
struct UnitShape {
    static constexpr int NB = B <= EPT ? EPT / B : 1;             // blocks per unit
    static constexpr int LPB = B <= EPT ? 1 : B / EPT;            // lanes per block
    static constexpr int BE = B <= EPT ? B : EPT;                 // elements of a block in one unit
    static constexpr int kChunk = K == 0 ? 1 : (K <= EPT ? K : EPT); // in-register rotation run
    static constexpr int kRotLanes = K > EPT ? K / EPT : 1;
    static_assert(LPB <= 32 && kRotLanes <= 32, "block or rotation wider than a warp");
};

// ---------------------------------------------------------------- ring of tiles
// BYTES_PER_UNIT bytes of input per unit (16, 32 or 64), UPS units per lane
// per tile.  All per-lane offsets are computed once; a tile that lies wholly
// inside the input is copied with one cp.async per 16-byte chunk at immediate
// offsets, only the last tile of the input takes the clamped path.
template <int BYTES_PER_UNIT, int UPS>
struct Ring {
    static constexpr int CPL = BYTES_PER_UNIT / 16;               // 16-byte chunks per lane per sub-tile
    static constexpr int SUB_BYTES = 32 * BYTES_PER_UNIT;         // one sub-tile
    static constexpr int TILE_BYTES = UPS * SUB_BYTES;
    static constexpr int NSTAGE = kRingBytesPerWarp / TILE_BYTES;
    static_assert(NSTAGE >= 2, "ring too small");
    static_assert(CPL == 1 || CPL == 2 || CPL == 4, "unsupported unit size");

    uint32_t base;                 // shared address of this warp's ring
    uint32_t wr[CPL];              // shared offset (in a sub-tile) of the chunk this lane copies, per c
    uint32_t rd[CPL];              // shared offset (in a sub-tile) of this lane's c-th chunk

    // smem chunk of global chunk j of a sub-tile: an XOR swizzle, constant over
    // each aligned group of 8 chunks, that keeps conflict free (8 lanes of a
    // 128-bit access cover the 8 distinct 16-byte bank groups) the contiguous
    // copies, the per-lane reads of a unit and, with 4 chunks per lane, the
    // reads of the 128-element run layout below: group m = (j / 8) mod 4 is
    // XORed with m ^ ((m & 2) << 1), i.e. 0, 1, 6, 7.
    static __device__ __forceinline__ int swz(int j)
    {
        if constexpr (CPL == 1) return j;
        if constexpr (CPL == 2) return j ^ ((j >> 3) & 1);
        const int m = (j >> 3) & 3;
        return j ^ (m ^ ((m & 2) << 1));
    }

    // runs128 (4 chunks per lane only): the lanes 4g .. 4g+3 that own the
    // 128-element run g of a tile read it interleaved, lane 4g + c getting the
    // chunks (8 elements each) 4j + c of the run, j = 0..3, in place of its own
    // unit's four; see unit_sums.
    __device__ __forceinline__ Ring(uint32_t b, int lane, bool runs128 = false) : base(b)
    {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            wr[c] = 16u * (uint32_t)swz(lane + 32 * c);
            const int j = (CPL == 4 && runs128) ? 16 * (lane >> 2) + 4 * c + (lane & 3) : CPL * lane + c;
            rd[c] = 16u * (uint32_t)swz(j);
        }
    }

    // Start the copies of the tile at byte offset off of src (nbytes long in
    // all) into stage s.  Bytes at or past nbytes are never read: a chunk
    // that straddles the end copies its valid prefix, and the rest, like every
    // chunk past the end, is zero-filled.
    // With EF the copies allocate their L2 lines evict-first (policy pol).
    template <bool EF = false>
    __device__ __forceinline__ void issue(const uint8_t* __restrict__ src, int64_t nbytes, int64_t off, int s,
                                          int lane, uint64_t pol = 0) const
    {
        const uint32_t sb = base + (uint32_t)(s * TILE_BYTES);
        const uint8_t* g = src + off + 16 * lane;
        if (off + TILE_BYTES <= nbytes) {
#pragma unroll
            for (int h = 0; h < UPS; ++h)
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    const uint32_t d = sb + (uint32_t)(h * SUB_BYTES) + wr[c];
                    if constexpr (EF) cp_async16(d, g + h * SUB_BYTES + 512 * c, 16u, pol);
                    else cp_async16(d, g + h * SUB_BYTES + 512 * c, 16u);
                }
        } else {
#pragma unroll
            for (int h = 0; h < UPS; ++h)
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    const int64_t o = off + h * SUB_BYTES + 512 * c + 16 * lane;
                    const int64_t left = nbytes - o;
                    const uint32_t cnt = left >= 16 ? 16u : (left > 0 ? (uint32_t)left : 0u);
                    cp_async16(sb + (uint32_t)(h * SUB_BYTES) + wr[c], cnt ? (const void*)(src + o) : (const void*)src,
                               cnt);
                }
        }
    }

    // This lane's unit of sub-tile h of stage s, as 32-bit words.
    __device__ __forceinline__ void read(int s, int h, uint32_t (&w)[BYTES_PER_UNIT / 4]) const
    {
        const uint32_t sb = base + (uint32_t)(s * TILE_BYTES + h * SUB_BYTES);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const uint4 v = lds128(sb + rd[c]);
            w[4 * c + 0] = v.x;
            w[4 * c + 1] = v.y;
            w[4 * c + 2] = v.z;
            w[4 * c + 3] = v.w;
        }
    }
};

// This warp's ring; K: the rotation of the kernel's units (a rotation wider
// than a unit reads its runs interleaved, see unit_sums).
template <typename R, int K = 0>
__device__ __forceinline__ R warp_ring(uint8_t* smem)
{
    return R((uint32_t)__cvta_generic_to_shared(smem) + (uint32_t)((threadIdx.x >> 5) * kRingBytesPerWarp),
             threadIdx.x & 31, K > EPT);
}

// Shared-memory scratch of a rotation wider than a unit (the lane transpose
// in unit_sums): 131 16-byte chunks per warp, in the dynamic shared memory
// right after the ring.  A kernel that instantiates such a rotation launches
// with ring_smem_bytes<K>() of dynamic shared memory (or more, other regions
// following the scratch).
constexpr int kRotScratchBytesPerWarp = 131 * 16;

template <int K>
__host__ __device__ constexpr int rot_scratch_bytes()
{
    return K > EPT ? kRotScratchBytesPerWarp * kWarps : 0;
}

template <int K>
__host__ __device__ constexpr int ring_smem_bytes()
{
    return kRingBytesPerCta + rot_scratch_bytes<K>();
}

extern __shared__ __align__(128) uint8_t smem_dynamic[];

__device__ __forceinline__ uint32_t rot_scratch()
{
    return (uint32_t)__cvta_generic_to_shared(smem_dynamic) + (uint32_t)kRingBytesPerCta +
           (uint32_t)((threadIdx.x >> 5) * kRotScratchBytesPerWarp);
}

// Ring pipeline driver: calls body(tile, stage) for every tile of this warp,
// with the tile's input resident in the ring; issue(tile, stage) starts the
// copies of a tile.  NSTAGE - 1 tiles are in flight.  ring_prime issues the
// first NSTAGE - 1 tiles, ring_run the rest while it runs the body: a kernel can
// prime its ring first and overlap the copies' latency with its own set-up.
template <int NS, typename Issue>
__device__ __forceinline__ void ring_prime(int64_t n_tiles, int64_t warp, int64_t n_warps, Issue&& issue)
{
    int64_t t_issue = warp;
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) {
        if (t_issue < n_tiles) issue(t_issue, s);
        cp_async_commit();
        t_issue += n_warps;
    }
}

template <int NS, typename Issue, typename Body>
__device__ __forceinline__ void ring_run(int64_t n_tiles, int64_t warp, int64_t n_warps, Issue&& issue, Body&& body)
{
    int64_t t_issue = warp + (int64_t)(NS - 1) * n_warps;
    int stage = 0;
    for (int64_t t = warp; t < n_tiles; t += n_warps) {
        const int s_new = stage == 0 ? NS - 1 : stage - 1;          // the slot read last iteration
        if (t_issue < n_tiles) issue(t_issue, s_new);
        cp_async_commit();
        t_issue += n_warps;
        cp_async_wait<NS - 1>();                                   // tile t has landed (own copies)
        __syncwarp();                                              // ... and every lane's copies
        body(t, stage);
        stage = stage + 1 == NS ? 0 : stage + 1;
        __syncwarp();                                              // slot may be refilled next iteration
    }
    cp_async_wait_all();
}

template <int NS, typename Issue, typename Body>
__device__ __forceinline__ void stream_tiles_with(int64_t n_tiles, int64_t warp, int64_t n_warps, Issue&& issue,
                                                  Body&& body)
{
    ring_prime<NS>(n_tiles, warp, n_warps, issue);
    ring_run<NS>(n_tiles, warp, n_warps, issue, body);
}

// The same over one contiguous input of nbytes bytes, tile t at byte t * TILE_BYTES.
// EF: the copies allocate their L2 lines evict-first (policy pol).
template <bool EF = false, typename R, typename Body>
__device__ __forceinline__ void stream_tiles(const R& ring, const uint8_t* __restrict__ src, int64_t nbytes,
                                             int64_t n_tiles, int64_t warp, int64_t n_warps, int lane,
                                             Body&& body, uint64_t pol = 0)
{
    stream_tiles_with<R::NSTAGE>(
        n_tiles, warp, n_warps,
        [&](int64_t t, int s) { ring.template issue<EF>(src, nbytes, t * R::TILE_BYTES, s, lane, pol); }, body);
}

using XRing = Ring<2 * EPT, 1>;                                  // one bf16 unit per lane per tile

// bf16 words -> fp32 pairs (exact widening; shift for the low half, a
// mixed-precision add for the high half, both on the floating-point pipe).
__device__ __forceinline__ void unpack_unit(const uint32_t (&w)[EPT / 2], f32x2 (&p)[EPT / 2])
{
#pragma unroll
    for (int k = 0; k < EPT / 2; ++k) p[k] = pk(bf16_lo(w[k]), bf16_hi_fp(w[k]));
}

// Lane transpose of the 128-element runs, half a unit at a time.  Lane
// L = 4g + c holds in p[4j + i] the pairs of elements 32j + 8c + 2i, +1 of run
// g (row j of the run as 4 rows of 32, its 8-element column c); afterwards
// lane 4g + j holds in p[4c + i] those of row j, columns c = 0..3: its own
// 32 consecutive elements.  Round h moves pairs i = 2h, 2h + 1 through
// scratch chunk R + 33 c for (row R = 4g + j of the warp, column c): every
// 16-byte store (fixed j) and load (fixed c) of 8 lanes hits 8 distinct bank
// groups, and each round refills exactly the registers it sent.  (Both halves
// at once, through two scratch regions and one barrier, measured slower.)
__device__ __forceinline__ void transpose_runs128(f32x2 (&p)[EPT / 2], int lane, uint32_t scr)
{
    const uint32_t rd = scr + 16u * (uint32_t)lane;              // row L, column c at + 528 c
    const uint32_t wr = rd + 512u * (uint32_t)(lane & 3);        // row 4g + j at + 16 j, column c
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        __syncwarp();                                            // the scratch's last readers are done
#pragma unroll
        for (int j = 0; j < 4; ++j) sts_pairs(wr + 16u * j, p[4 * j + 2 * h], p[4 * j + 2 * h + 1]);
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) lds_pairs(rd + 528u * c, p[4 * c + 2 * h], p[4 * c + 2 * h + 1]);
    }
}

// The Sylvester sums of a unit's runs of K elements (K > 0).  The odd
// positions come out negated (see unpack_fwht2); only magnitudes are read
// from the result, or normalise_signed restores the signs.
// K <= 32: the runs lie inside the unit, all in registers.
// K = 128: a run spans 4 lanes.  The ring hands each lane the run's
// interleaved chunks (Ring, runs128), so that the stages of element bits 0-2
// and 5-6 run in registers; a transpose through shared memory (the warp's
// rot_scratch) gives each lane its own 32 elements back, and the stages of
// bits 3-4 run in registers too.  Same sums as the stages in bit order, with
// the roundings of a different order.
template <int K>
__device__ __forceinline__ void unit_sums(const uint32_t (&w)[EPT / 2], f32x2 (&p)[EPT / 2], int lane)
{
    static_assert(K >= 2 && (K <= EPT || K == 4 * EPT), "rotation runs of 2..32 or 128 elements");
    unpack_fwht2<EPT>(w, p);
    fwht_inreg<EPT, (K < EPT ? K : EPT), false>(p);
    if constexpr (K > EPT) {
        transpose_runs128(p, lane, rot_scratch());
        fwht_inreg<EPT, EPT, false, 8>(p);
    }
}

// y = s / sqrt(K) rounded to fp32, the odd positions' signs restored by
// multiplying them by the negated constant.  K = 16: 1/sqrt(K) = 1/4 is exact,
// one product per value.  K = 32, 128: the constant is split as c_hi + c_lo
// (both fp32, from the fp64 value) and y = fp32(s c_hi + fp32(s c_lo)), the
// fp32 value nearest to s / sqrt(K) except within ~2^-47 (relative) of a
// rounding midpoint (a single product by c_hi would add up to 0.14 ulp, and
// with it codes that differ from the exact rotation's at E2M1 ties).  Every
// rounding adds +0 last, which leaves non-zero values as they are and makes
// every zero +0: an exact cancellation in a negated position would otherwise
// come out as -0, while a zero of the exact rotation (a sum that starts from
// +0) is +0.
template <int K>
__device__ __forceinline__ void normalise_signed(f32x2 (&p)[EPT / 2], float c_hi, float c_lo)
{
    const f32x2 hi = pk(c_hi, -c_hi), z = pk(0.0f, 0.0f);
    if constexpr (K == 16) {
#pragma unroll
        for (int k = 0; k < EPT / 2; ++k) p[k] = fma2(p[k], hi, z);
    } else {
        const f32x2 lo = pk(c_lo, -c_lo);
#pragma unroll
        for (int k = 0; k < EPT / 2; ++k) p[k] = fma2(p[k], hi, fma2(p[k], lo, z));
    }
}

// A unit's values for quantization: the widened bf16 inputs (K = 0), or their
// rotation by H_K / sqrt(K) over runs of K elements.
template <int K>
__device__ __forceinline__ void load_unit(const uint32_t (&w)[EPT / 2], f32x2 (&p)[EPT / 2], int lane, float c_hi,
                                          float c_lo)
{
    if constexpr (K == 0) {
        unpack_unit(w, p);
    } else {
        unit_sums<K>(w, p, lane);
        normalise_signed<K>(p, c_hi, c_lo);
    }
}

// Absolute maximum of the CNT values of p (CNT even).
template <int CNT>
__device__ __forceinline__ float pairs_absmax(const f32x2* p)
{
    float a, b, m = 0.0f;
#pragma unroll
    for (int k = 0; k < CNT / 2; ++k) {
        upk(p[k], a, b);
        m = amax3(a, b, m);
    }
    return m;
}

// Per-block absolute maximum of a unit (combined across lanes for wide blocks).
template <int B, int K>
__device__ __forceinline__ void block_max(const f32x2 (&p)[EPT / 2], float (&m)[UnitShape<B, K>::NB])
{
    using S = UnitShape<B, K>;
#pragma unroll
    for (int bi = 0; bi < S::NB; ++bi) m[bi] = pairs_absmax<S::BE>(p + bi * S::BE / 2);
    if constexpr (S::LPB > 1) m[0] = group_max<S::LPB>(m[0]);
}

// The same maxima straight from the bf16 words of an unrotated unit: packed
// two-wide magnitude maxima, then the larger half (exact).
template <int B>
__device__ __forceinline__ void block_max_words(const uint32_t (&w)[EPT / 2], float (&m)[UnitShape<B, 0>::NB])
{
    using S = UnitShape<B, 0>;
    constexpr int WPB = S::BE / 2;                                  // words of a block in this unit
#pragma unroll
    for (int bi = 0; bi < S::NB; ++bi) {
        uint32_t a = w[bi * WPB];
#pragma unroll
        for (int k = 1; k < WPB; ++k) a = bf16x2_absmax(a, w[bi * WPB + k]);
        m[bi] = bf16x2_absmax_f32(a);
    }
    if constexpr (S::LPB > 1) m[0] = group_max<S::LPB>(m[0]);
}

template <int LANES>
__device__ __forceinline__ float group_sum(float s)
{
#pragma unroll
    for (int d = 1; d < LANES; d <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, d));
    return s;
}

// Per-CTA reduction of four fp64 accumulators into partials[blockIdx.x][4], in a
// fixed order (warp butterflies, then warps in index order): deterministic.
template <int NT = kThreads>
__device__ __forceinline__ void cta_partials(double a0, double a1, double a2, double a3, double* partials)
{
    constexpr int NW = NT / 32;
    __shared__ double red[NW][4];
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
        a0 += __shfl_xor_sync(0xffffffffu, a0, d);
        a1 += __shfl_xor_sync(0xffffffffu, a1, d);
        a2 += __shfl_xor_sync(0xffffffffu, a2, d);
        a3 += __shfl_xor_sync(0xffffffffu, a3, d);
    }
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) {
        red[wid][0] = a0;
        red[wid][1] = a1;
        red[wid][2] = a2;
        red[wid][3] = a3;
    }
    __syncthreads();
    if (threadIdx.x < 4) {
        double s = 0.0;
        for (int k = 0; k < NW; ++k) s += red[k][threadIdx.x];
        partials[(int64_t)blockIdx.x * 4 + threadIdx.x] = s;
    }
}

// The tensor terms from the per-CTA partials, inside the kernel that wrote
// them: every CTA counts itself done on a counter (after making its partials
// visible); the CTA that finishes last sums partials[0..gridDim.x) in index
// order (deterministic), writes terms[i] = sum / n, and atomicInc's wrap-around
// leaves the counter at 0 for the next call.  The counter must be 0 when the
// kernel starts.
template <int NT = kThreads>
__device__ __forceinline__ void finish_partials(const double* partials, unsigned int* done, int64_t n, double* terms)
{
    constexpr int NW = NT / 32;
    __shared__ bool last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicInc(done, gridDim.x - 1u) == gridDim.x - 1u;
    __syncthreads();
    if (!last) return;
    __threadfence();
    __shared__ double red[NW][4];
    double s[4] = {0.0, 0.0, 0.0, 0.0};
    for (int i = threadIdx.x; i < (int)gridDim.x; i += NT)
#pragma unroll
        for (int k = 0; k < 4; ++k) s[k] += __ldcg(partials + (int64_t)i * 4 + k);
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1)
#pragma unroll
        for (int k = 0; k < 4; ++k) s[k] += __shfl_xor_sync(0xffffffffu, s[k], d);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0)
#pragma unroll
        for (int k = 0; k < 4; ++k) red[wid][k] = s[k];
    __syncthreads();
    if (threadIdx.x < 4) {
        double t = 0.0;
        for (int w = 0; w < NW; ++w) t += red[w][threadIdx.x];
        terms[threadIdx.x] = t / (double)n;
    }
}

// Grid values of the 8 nibbles of a code word as 4 fp32 pairs (exact).
__device__ __forceinline__ void decode8(uint32_t cw, f32x2 (&g)[4])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a, b;
        e2m1_unpack2((cw >> (8 * j)) & 0xffu, a, b);
        g[j] = pk(a, b);
    }
}

// E2M1 codes of 4 pairs -> one code word (low nibble = even element).
__device__ __forceinline__ uint32_t pack_pairs(f32x2 p0, f32x2 p1, f32x2 p2, f32x2 p3)
{
    float a0, b0, a1, b1, a2, b2, a3, b3;
    upk(p0, a0, b0);
    upk(p1, a1, b1);
    upk(p2, a2, b2);
    upk(p3, a3, b3);
    return e2m1_pack8(a0, b0, a1, b1, a2, b2, a3, b3);
}

// E2M1 codes of 4 pairs -> code word, and the grid values decoded back (f16x2 per pair).
__device__ __forceinline__ uint32_t pack_pairs_dec(f32x2 p0, f32x2 p1, f32x2 p2, f32x2 p3, uint32_t (&h)[4])
{
    float a0, b0, a1, b1, a2, b2, a3, b3;
    upk(p0, a0, b0);
    upk(p1, a1, b1);
    upk(p2, a2, b2);
    upk(p3, a3, b3);
    return e2m1_pack8_dec(a0, b0, a1, b1, a2, b2, a3, b3, h);
}

// Codes of 4 pairs with correctly rounded quotients v / s (s != 0) by
// division: the fallback for scales outside the range the remainder
// correction serves (extreme per-tensor scales), kept out of line.
static __device__ __noinline__ uint32_t pack_pairs_div(f32x2 p0, f32x2 p1, f32x2 p2, f32x2 p3, float s)
{
    float a[8];
    upk(p0, a[0], a[1]);
    upk(p1, a[2], a[3]);
    upk(p2, a[4], a[5]);
    upk(p3, a[6], a[7]);
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = __fdiv_rn(a[j], s);
    return e2m1_pack8(a[0], a[1], a[2], a[3], a[4], a[5], a[6], a[7]);
}

// Per-tensor table of the UE block scales, tab[c] = {S, R}: S = fp32(decode(c)
// G) and R = fp32(1/S) correctly rounded; R = 0 for S = 0 (a zero-rounded
// block), R = +inf for S outside [2^-100, 2^100] or a NaN code, which makes
// the block divide instead (see unit_scales).
template <int FMT>
__device__ __forceinline__ void fill_scale_table(float2* tab, float G)
{
    for (int c = threadIdx.x; c < 256; c += blockDim.x) {
        float S;
        if (FMT == kUE4M3) S = c < 127 ? __fmul_rn(ue4m3_decode((uint32_t)c), G) : __uint_as_float(0x7fc00000u);
        else S = c < 255 ? __fmul_rn(ue5m3_decode((uint32_t)c), G) : __uint_as_float(0x7fc00000u);
        float R;
        if (S == 0.0f) R = 0.0f;
        else if (S >= kDivLo && S <= kDivHi) R = __frcp_rn(S);
        else R = __uint_as_float(0x7f800000u);
        tab[c] = make_float2(S, R);
    }
}

// Scales of the NB blocks of a unit ("max" rule): scale bytes, S and R =
// fp32(1/S).  E8M0: S = 2^(floor(log2 m) - 2), R exact.  UE4M3 / UE5M3: the
// byte is the code nearest the correctly rounded quotient fp32(m / fp32(6G))
// (two blocks per instruction), S and R come from the table.  Returns false
// when some block must divide its elements: fp32(6G) or S outside the range
// of the remainder correction, or a quotient m / S beyond 2^60.
template <int FMT, int NB>
__device__ __forceinline__ bool unit_scales(const float (&m)[NB], const ScaleConsts& kc, const float2* tab,
                                            uint32_t (&code)[NB], float (&S)[NB], float (&R)[NB])
{
    if constexpr (FMT == kE8M0) {
#pragma unroll
        for (int bi = 0; bi < NB; ++bi) {
            code[bi] = e8m0_from_amax(m[bi]);
            S[bi] = e8m0_decode(code[bi]);
            R[bi] = e8m0_inverse(code[bi]);
        }
        return true;
    } else {
        bool fast = kc.denom_ok;
#pragma unroll
        for (int bi = 0; bi < NB; bi += 2) {
            const float m1 = bi + 1 < NB ? m[bi + 1] : m[bi];
            float s0, s1;
            if (kc.denom_ok) {
                upk(div2_cr(pk(m[bi], m1), pk(kc.rdenom, kc.rdenom), pk(-kc.denom, -kc.denom)), s0, s1);
            } else {
                s0 = __fdiv_rn(m[bi], kc.denom);
                s1 = __fdiv_rn(m1, kc.denom);
            }
            uint32_t c0, c1;
            if constexpr (FMT == kUE4M3) {
                const uint32_t cc = ue4m3_encode2(s0, s1);
                c0 = cc & 0xffu;
                c1 = cc >> 8;
            } else {
                c0 = ue5m3_encode(s0);
                c1 = ue5m3_encode(s1);
            }
            code[bi] = c0;
            if (bi + 1 < NB) code[bi + 1] = c1;
        }
#pragma unroll
        for (int bi = 0; bi < NB; ++bi) {
            const float2 e = tab[code[bi]];
            S[bi] = e.x;
            R[bi] = e.y;
            fast = fast && (__fmul_rn(m[bi], e.y) <= kQuotMax);
        }
        return fast;
    }
}

// Largest dequantized magnitude of a block, |v| of its maximum m: the grid
// value that fp32(m / S) rounds to, times S.  For a UE scale with a normal
// code (byte >= 8: 3 significant bits), when fp32(6G) and S are in the
// normal range (`fast`), decode(s) is within 2^-4 (relative) of m / fp32(6G),
// so m / S lies in [5.6, 6.5] and always rounds to 6.  E8M0 scales are powers
// of two, so m * (1/S) is the exact quotient.  Other UE blocks divide.
template <int FMT>
__device__ __forceinline__ float block_vmax(float m, float S, float r_mid, uint32_t code, bool fast)
{
    if (S == 0.0f) return 0.0f;
    if constexpr (FMT == kE8M0) {
        return __fmul_rn(e2m1_grid_value(__fmul_rn(m, r_mid)), S);
    } else {
        if (fast && code >= 8u) return __fmul_rn(6.0f, S);
        return __fmul_rn(e2m1_grid_value(__fdiv_rn(m, S)), S);
    }
}

// ---------------------------------------------------------------- quantize
struct QuantParams {
    const uint16_t* x;     // bf16 bits
    int64_t n;             // elements
    uint8_t* codes;        // n/2 bytes
    uint8_t* scales;       // n/B bytes
    const float* gsrc;     // per-tensor scale G (nullptr: G = 1)
    float c_hi, c_lo;      // 1/sqrt(K) split in two fp32 parts
    float* block_mse;      // fused MSE: n/B floats or nullptr
    double* partials;      // fused MSE: [gridDim.x][4]
    unsigned int* done;    // fused MSE: completion counter (0 at launch, left 0)
    double* terms;         // fused MSE: the four tensor terms
    float* gdst;           // G from the tensor maximum: *gsrc is that maximum, G is written here
    uint16_t* y;           // fused MSE with dequantized output: n bf16 values
    int below, above;      // scale search: codes tried below / above the max-rule code
    int64_t sf_cols;       // > 0: scale bytes in the block-scaled MMA layout, sf_cols = cols / B
    int64_t sf_kt;         //   ... with sf_kt = ceil(sf_cols / 4) 512-byte atoms per 128-row block
};

// Offset of scale byte (row r, block column j) in the block-scaled MMA layout:
// 512-byte atoms of 128 rows x 4 consecutive block scales, atom (r / 128,
// j / 4) at ((r / 128) sf_kt + j / 4) * 512; inside, row r % 128 = 32 g + i
// holds its 4 bytes at i * 16 + g * 4, so each 32-bit word is one row's 4
// scales and each 16-byte line the words of rows i, i + 32, i + 64, i + 96.
__device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t j, int64_t sf_kt)
{
    return (((r >> 7) * sf_kt + (j >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (j & 3);
}

// Store a unit's code word (16 bytes; with EF evict-first in L2, for codes
// that nothing reads again in the step) and its blocks' scale bytes; a unit
// that reaches past n stores only its valid prefix.
// SF = false: the caller never asks for the block-scaled MMA layout (sf_cols = 0).
template <int B, int K, bool EF, bool SF = true>
__device__ __forceinline__ void store_unit(const QuantParams& p, int64_t u, const uint32_t (&cw)[EPT / 8],
                                           const uint32_t (&code)[UnitShape<B, K>::NB], int lane, uint64_t pol)
{
    using S = UnitShape<B, K>;
    constexpr int NB = S::NB;
    const int64_t e0 = u * EPT;
    if (e0 >= p.n) return;
    uint8_t* cdst = p.codes + e0 / 2;
    if (e0 + EPT <= p.n) {
        if constexpr (EF) stg128(cdst, cw[0], cw[1], cw[2], cw[3], pol);
        else stg128(cdst, cw[0], cw[1], cw[2], cw[3]);
    } else {
        const int nbytes = (int)((p.n - e0) / 2);
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (4 * k + j < nbytes) cdst[4 * k + j] = (uint8_t)(cw[k] >> (8 * j));
    }
    if (SF && p.sf_cols > 0) {
        // the block-scaled MMA layout: a unit's blocks lie in one row
        const int64_t g0 = e0 / B;
        const int64_t r = g0 / p.sf_cols, j0 = g0 - r * p.sf_cols;
        if constexpr (S::LPB > 1) {
            if ((lane % S::LPB) == 0) p.scales[mma_scale_offset(r, j0, p.sf_kt)] = (uint8_t)code[0];
        } else {
            const int64_t nblk = p.n / B;
#pragma unroll
            for (int bi = 0; bi < NB; ++bi)
                if (g0 + bi < nblk) p.scales[mma_scale_offset(r, j0 + bi, p.sf_kt)] = (uint8_t)code[bi];
        }
    } else if constexpr (S::LPB > 1) {
        if ((lane % S::LPB) == 0) p.scales[e0 / B] = (uint8_t)code[0];
    } else {
        const int64_t b0 = e0 / B;
        const int64_t nblk = p.n / B;
        if (e0 + EPT <= p.n) {
            if constexpr (NB == 1) {
                p.scales[b0] = (uint8_t)code[0];
            } else if constexpr (NB == 2) {
                *reinterpret_cast<uint16_t*>(p.scales + b0) = (uint16_t)(code[0] | (code[1] << 8));
            } else {
                *reinterpret_cast<uint32_t*>(p.scales + b0) =
                    code[0] | (code[1] << 8) | (code[2] << 16) | (code[3] << 24);
            }
        } else {
#pragma unroll
            for (int bi = 0; bi < NB; ++bi)
                if (b0 + bi < nblk) p.scales[b0 + bi] = (uint8_t)code[bi];
        }
    }
}

// Scale, codes, MSE terms, dequantized values and stores of unit u, whose
// blocks' absolute maxima are m and whose (rotated) values are produced half
// by half: half(h, vh) fills vh with elements 16 h .. 16 h + 15 as 8 pairs
// (h = 0 then 1), so a caller can hold only half of the unit in registers.
template <int FMT, int B, int K, bool MSE, bool DQ, bool SF = true, typename Half>
__device__ __forceinline__ void quantize_halves(const QuantParams& p, int64_t u, Half&& half,
                                                const float (&m)[UnitShape<B, K>::NB], int lane,
                                                const ScaleConsts& kc, const float2* tab, float nz,
                                                double (&acc)[3], uint64_t pol)
{
    using S = UnitShape<B, K>;
    constexpr int NB = S::NB, BE = S::BE;
    float sc[NB], rm[NB];
    uint32_t code[NB];
    const bool exact = unit_scales<FMT, NB>(m, kc, tab, code, sc, rm);

    // ---- codes, one 8-element word at a time; each word's code bytes are also
    // decoded straight back for the MSE, whose squared errors are taken right
    // away (three-term split of "Finer is better?": v_i = fp32(decode(code_i) * S))
    uint32_t cw[EPT / 8];
    uint32_t ypend[4];                           // bf16 words of the previous (even) word, stored in pairs
    f32x2 bsum[NB];
#pragma unroll
    for (int bi = 0; bi < NB; ++bi) bsum[bi] = pk(0.0f, 0.0f);
    // A zero-rounded block (UE scale 0) stores plain 0x0 nibbles, which decode to
    // +0.  Its quotients y * 0 are zeros that keep y's sign, so its code words are
    // masked to 0, and its products g * 0 get the addend +0 (which makes them +0),
    // where every other block's get -0 (fma(g, S, -0) is the rounded product
    // fp32(g S), sign of zero included): its dequantized values go out as +0 and
    // each of its errors is y itself.
    uint32_t zmask[NB];
    f32x2 zadd[NB];
#pragma unroll
    for (int bi = 0; bi < NB; ++bi) {
        zmask[bi] = (FMT != kE8M0 && sc[bi] == 0.0f) ? 0u : 0xffffffffu;
        const float a = __uint_as_float(__float_as_uint(nz) & zmask[bi]);
        zadd[bi] = pk(a, a);
    }
    f32x2 vh[EPT / 4];
#pragma unroll
    for (int k = 0; k < EPT / 8; ++k) {
        const int bi = (8 * k) / BE;
        if ((k & 1) == 0) half(k >> 1, vh);
        const f32x2* vk = vh + 4 * (k & 1);
        uint32_t h[4];
        if constexpr (FMT == kE8M0) {
            // S is a power of two: y * (1/S) is the quotient itself.
            const f32x2 r = pk(rm[bi], rm[bi]);
            cw[k] = pack_pairs_dec(mul2(vk[0], r), mul2(vk[1], r), mul2(vk[2], r), mul2(vk[3], r), h);
        } else {
            if (exact) {
                // correctly rounded quotients y / S (remainder correction), then the
                // hardware E2M1 rounding (nearest, ties to the even code, saturating)
                const f32x2 R2 = pk(rm[bi], rm[bi]), nS2 = pk(-sc[bi], -sc[bi]);
                cw[k] = pack_pairs_dec(div2_cr(vk[0], R2, nS2), div2_cr(vk[1], R2, nS2), div2_cr(vk[2], R2, nS2),
                                       div2_cr(vk[3], R2, nS2), h) &
                        zmask[bi];
            } else {
                // extreme scales: correctly rounded divisions
                cw[k] = sc[bi] != 0.0f ? pack_pairs_div(vk[0], vk[1], vk[2], vk[3], sc[bi]) : 0u;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t hh;
                    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(hh) : "r"((cw[k] >> (8 * j)) & 0xffu));
                    h[j] = hh;
                }
            }
        }
        if constexpr (MSE) {
            const f32x2 s2 = pk(sc[bi], sc[bi]);
            uint32_t yw[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 hh = *reinterpret_cast<__half2*>(&h[j]);
                const f32x2 g = pk(__low2float(hh), __high2float(hh));
                const f32x2 vq = fma2(g, s2, zadd[bi]);              // v = fp32(g S); +0 in a zero-rounded block
                const f32x2 d = sub2(vk[j], vq);                     // y - v
                bsum[bi] = fma2(d, d, bsum[bi]);
                if constexpr (DQ) {
                    float a, b;
                    upk(vq, a, b);
                    __nv_bfloat162 hb = __floats2bfloat162_rn(a, b);
                    yw[j] = *reinterpret_cast<uint32_t*>(&hb);
                }
            }
            if constexpr (DQ) {
                // the dequantized values of this word, as fp4q_dequantize writes them;
                // two words (32 bytes) per store
                const int64_t ew = u * EPT + 8 * k;
                if (u * EPT + EPT <= p.n) {
                    if ((k & 1) == 0) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) ypend[j] = yw[j];
                    } else {
                        stg256(p.y + ew - 8, ypend[0], ypend[1], ypend[2], ypend[3], yw[0], yw[1], yw[2], yw[3],
                               pol);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if (ew + 2 * j < p.n) p.y[ew + 2 * j] = (uint16_t)(yw[j] & 0xffffu);
                        if (ew + 2 * j + 1 < p.n) p.y[ew + 2 * j + 1] = (uint16_t)(yw[j] >> 16);
                    }
                }
            }
        }
    }
    if constexpr (MSE) {
        float tot = 0.0f, mx = 0.0f, zr = 0.0f;
#pragma unroll
        for (int bi = 0; bi < NB; ++bi) {
            float se, so;
            upk(bsum[bi], se, so);
            float s = __fadd_rn(se, so);
            if constexpr (S::LPB > 1) s = group_sum<S::LPB>(s);
            const float vmax = block_vmax<FMT>(m[bi], sc[bi], rm[bi], code[bi], exact);
            const int64_t eb = u * EPT + (int64_t)bi * BE;
            const bool leader = (S::LPB == 1) || ((lane % S::LPB) == 0);
            if (leader && eb < p.n) {
                if (p.block_mse) p.block_mse[eb / B] = __fmul_rn(s, 1.0f / (float)B);
                tot = __fadd_rn(tot, s);
                if (vmax == 0.0f) {
                    zr = __fadd_rn(zr, s);                  // every v of the block is 0
                } else {
                    const float dm = __fsub_rn(m[bi], vmax);   // the maximum rounds to the largest |v|
                    mx = __fmaf_rn(dm, dm, mx);
                }
            }
        }
        acc[0] += (double)tot;
        acc[1] += (double)mx;
        if (zr != 0.0f) acc[2] += (double)zr;
    }

    // ---- stores
    store_unit<B, K, DQ, SF>(p, u, cw, code, lane, pol);
}

// The same for a unit held whole in registers.
template <int FMT, int B, int K, bool MSE, bool DQ, bool SF = true>
__device__ __forceinline__ void quantize_values(const QuantParams& p, int64_t u, const f32x2 (&v)[EPT / 2],
                                                const float (&m)[UnitShape<B, K>::NB], int lane,
                                                const ScaleConsts& kc, const float2* tab, float nz,
                                                double (&acc)[3], uint64_t pol)
{
    quantize_halves<FMT, B, K, MSE, DQ, SF>(
        p, u,
        [&](int h, f32x2 (&vh)[EPT / 4]) {
#pragma unroll
            for (int j = 0; j < EPT / 4; ++j) vh[j] = v[(EPT / 4) * h + j];
        },
        m, lane, kc, tab, nz, acc, pol);
}

// SF as for store_unit; c_hi, c_lo: the rotation constant (p's own, or one a
// batch of tensors shares).
template <int FMT, int B, int K, bool MSE, bool DQ, bool SF = true>
__device__ __forceinline__ void quantize_unit(const QuantParams& p, int64_t u, const uint32_t (&w)[EPT / 2],
                                              int lane, const ScaleConsts& kc, const float2* tab, float nz,
                                              double (&acc)[3], uint64_t pol, float c_hi, float c_lo)
{
    using S = UnitShape<B, K>;
    f32x2 v[EPT / 2];
    load_unit<K>(w, v, lane, c_hi, c_lo);
    float m[S::NB];
    if constexpr (K == 0) block_max_words<B>(w, m);
    else block_max<B, K>(v, m);
    quantize_values<FMT, B, K, MSE, DQ, SF>(p, u, v, m, lane, kc, tab, nz, acc, pol);
}

template <int FMT, int B, int K, bool MSE, bool DQ>
__device__ __forceinline__ void quantize_unit(const QuantParams& p, int64_t u, const uint32_t (&w)[EPT / 2],
                                              int lane, const ScaleConsts& kc, const float2* tab, float nz,
                                              double (&acc)[3], uint64_t pol)
{
    quantize_unit<FMT, B, K, MSE, DQ, true>(p, u, w, lane, kc, tab, nz, acc, pol, p.c_hi, p.c_lo);
}

// Two CTAs per SM (up to 128 registers) unless the kernel fits three without
// spilling: measured, spills in the UE and fused variants cost more than the
// extra warps gain.
template <int FMT, int B, int K, bool MSE, bool DQ = false>
__global__ void __launch_bounds__(kThreads, (MSE || FMT != kE8M0) ? 2 : 3) quantize_kernel(QuantParams p)
{
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem_ring[];
    const int lane = threadIdx.x & 31;
    const int64_t n_tiles = (p.n + 32 * EPT - 1) / (32 * EPT);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const XRing ring = warp_ring<XRing, K>(smem_ring);

    // Evict-first in L2 for what the step does not read again, so that it does
    // not push out lines that are: x where this is its last read (MSE fused), and
    // the codes and dequantized values of the fused dequantizing kernel.
    const uint64_t pol = l2_evict_first();
    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.x);
    auto issue = [&](int64_t t, int s) { ring.template issue<MSE>(src, 2 * p.n, t * XRing::TILE_BYTES, s, lane, pol); };
    // The first tiles load during the set-up below, except in the rotated UE-scale
    // kernels: their loop is the most register-bound, and starting the copies
    // earlier measured 2.5% slower there (1-2% faster elsewhere).
    constexpr bool kPrimeEarly = FMT == kE8M0 || K == 0;
    if constexpr (kPrimeEarly) ring_prime<XRing::NSTAGE>(n_tiles, warp, n_warps, issue);

    float G = 1.0f;
    if (FMT != kE8M0 && p.gsrc != nullptr) {
        G = *p.gsrc;
        if (p.gdst != nullptr) {
            // per-tensor scale from the tensor maximum: amax / (6 * 448), 1 for an all-zero tensor
            G = G > 0.0f ? __fdiv_rn(G, 2688.0f) : 1.0f;
            if (blockIdx.x == 0 && threadIdx.x == 0) *p.gdst = G;
        }
    }
    const ScaleConsts kc = scale_consts(G);
    __shared__ float2 tab[256];                 // UE scales {S, 1/S} by code
    if constexpr (FMT != kE8M0) fill_scale_table<FMT>(tab, G);
    __syncthreads();
    // -0.0f from a value the compiler cannot see (n >= 0 at run time): an
    // fma with it rounds a product on its own and cannot be merged with the
    // subtraction that follows.
    const float nz = __uint_as_float(0x80000000u | (uint32_t)((uint64_t)p.n >> 63));
    double acc[3] = {0.0, 0.0, 0.0};        // squared errors: all, block maxima, zero-rounded blocks

    if constexpr (!kPrimeEarly) ring_prime<XRing::NSTAGE>(n_tiles, warp, n_warps, issue);
    ring_run<XRing::NSTAGE>(n_tiles, warp, n_warps, issue, [&](int64_t t, int s) {
        uint32_t w[EPT / 2];
        ring.read(s, 0, w);
        quantize_unit<FMT, B, K, MSE, DQ>(p, t * 32 + lane, w, lane, kc, tab, nz, acc, pol);
    });
    if constexpr (MSE) {
        cta_partials(acc[0], acc[0] - acc[1] - acc[2], acc[1], acc[2], p.partials);
        finish_partials(p.partials, p.done, p.n, p.terms);
    }
}

// ---------------------------------------------------------------- batched fused quantizer
// One launch quantizes up to kQuantBatch tensors of one format, block and
// rotation, each with its own per-tensor scale, outputs and MSE terms (what
// fp4q_quantize_mse_dequantize does for one).  Their ring tiles are laid end
// to end and every warp strides over all of them, so a layer's small
// projections pay one launch ramp and one tail instead of one each.
constexpr int kQuantBatch = 8;

struct QuantBatchParams {
    QuantParams t[kQuantBatch];          // per tensor: x, n, outputs, gsrc/gdst, partials, done, terms, y
    int32_t tile0[kQuantBatch + 1];      // first ring tile of each tensor; tile0[count] = all tiles
    int count;
};

// The last CTA to finish tensor c (a counter per tensor) sums its per-CTA
// partials into terms[c] = sum / n, one warp per tensor so that the tensors'
// sums run side by side (the same CTA is usually last for all of them).  A
// warp sums partials lane-strided and then by a fixed shuffle tree:
// deterministic.  Every CTA writes a partial for every tensor, zeros for
// tensors it never touched.
template <int NT = kThreads>
__device__ __forceinline__ void finish_partials_batch(const QuantBatchParams& P)
{
    constexpr int NW = NT / 32;
    __shared__ bool last[kQuantBatch];
    __threadfence();
    __syncthreads();
    if (threadIdx.x < (unsigned)P.count)
        last[threadIdx.x] = atomicInc(P.t[threadIdx.x].done, gridDim.x - 1u) == gridDim.x - 1u;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (int c = threadIdx.x >> 5; c < P.count; c += NW) {
        if (!last[c]) continue;                                    // warp-uniform
        __threadfence();
        const double* partials = P.t[c].partials;
        double s[4] = {0.0, 0.0, 0.0, 0.0};
        for (int i = lane; i < (int)gridDim.x; i += 32)
#pragma unroll
            for (int k = 0; k < 4; ++k) s[k] += __ldcg(partials + (int64_t)i * 4 + k);
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1)
#pragma unroll
            for (int k = 0; k < 4; ++k) s[k] += __shfl_xor_sync(0xffffffffu, s[k], d);
        if (lane == 0) {
            const int64_t n = P.t[c].n;
#pragma unroll
            for (int k = 0; k < 4; ++k) P.t[c].terms[k] = n > 0 ? s[k] / (double)n : 0.0;
        }
    }
}

template <int FMT, int B, int K>
__global__ void __launch_bounds__(kThreads, 2) quantize_batch_kernel(const __grid_constant__ QuantBatchParams P)
{
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem_ring[];
    __shared__ float2 tabs[FMT == kE8M0 ? 1 : kQuantBatch][256];   // UE scales {S, 1/S} by code, per tensor
    __shared__ float4 kcs[kQuantBatch];                            // per tensor: G, fp32(6G), 1/fp32(6G), in range
    __shared__ double wsum[kQuantBatch][kWarps][4];                // per tensor and warp: the MSE terms
    const int lane = threadIdx.x & 31;
    const int warp_in = threadIdx.x >> 5;
    const int32_t n_tiles = P.tile0[P.count];
    const int32_t warp = (int32_t)(blockIdx.x * (kThreads / 32)) + warp_in;
    const int32_t n_warps = (int32_t)(gridDim.x * (kThreads / 32));
    const XRing ring = warp_ring<XRing, K>(smem_ring);
    const uint64_t pol = l2_evict_first();

    // ---- the tiles of all tensors; a warp's tiles rise, so its tensors do too:
    // one cursor for the copies issued ahead, one for the tile being quantized
    struct Cursor {
        int c;
        int32_t t0, t1;
    };
    auto seek = [&](Cursor& k, int32_t t) {
        while (t >= k.t1) {
            ++k.c;
            k.t0 = k.t1;
            k.t1 = P.tile0[k.c + 1];
        }
    };
    Cursor ci{0, 0, P.tile0[1]}, cb{0, 0, P.tile0[1]};
    auto issue = [&](int64_t t, int s) {
        seek(ci, (int32_t)t);
        const QuantParams& q = P.t[ci.c];
        ring.template issue<true>(reinterpret_cast<const uint8_t*>(q.x), 2 * q.n,
                                  (int64_t)((int32_t)t - ci.t0) * XRing::TILE_BYTES, s, lane, pol);
    };
    // the first tiles load during the set-up, except in the rotated UE-scale kernels (as quantize_kernel)
    constexpr bool kPrimeEarly = FMT == kE8M0 || K == 0;
    if constexpr (kPrimeEarly) ring_prime<XRing::NSTAGE>(n_tiles, warp, n_warps, issue);

    // ---- per-tensor set-up: G (from the tensor maximum in FROM_AMAX mode), the
    // scale constants and the UE scale table, and zeroed MSE slots
    for (int c = 0; c < P.count; ++c) {
        float G = 1.0f;
        if (FMT != kE8M0 && P.t[c].gsrc != nullptr) {
            G = *P.t[c].gsrc;
            if (P.t[c].gdst != nullptr) {
                G = G > 0.0f ? __fdiv_rn(G, 2688.0f) : 1.0f;
                if (blockIdx.x == 0 && threadIdx.x == 0) *P.t[c].gdst = G;
            }
        }
        if (threadIdx.x == 0) {
            const ScaleConsts k = scale_consts(G);
            kcs[c] = make_float4(k.G, k.denom, k.rdenom, k.denom_ok ? 1.0f : 0.0f);
        }
        if constexpr (FMT != kE8M0) fill_scale_table<FMT>(tabs[c], G);
    }
    for (int i = threadIdx.x; i < kQuantBatch * kWarps * 4; i += kThreads) (&wsum[0][0][0])[i] = 0.0;
    __syncthreads();
    // -0.0f from a value the compiler cannot see (the tile count is >= 0)
    const float nz = __uint_as_float(0x80000000u | ((uint32_t)n_tiles >> 31));

    int cur = -1;
    ScaleConsts kc{};
    double acc[3] = {0.0, 0.0, 0.0};
    auto flush = [&]() {                                           // warp-uniform
        double a[4] = {acc[0], acc[0] - acc[1] - acc[2], acc[1], acc[2]};
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1)
#pragma unroll
            for (int k = 0; k < 4; ++k) a[k] += __shfl_xor_sync(0xffffffffu, a[k], d);
        if (lane == 0)
#pragma unroll
            for (int k = 0; k < 4; ++k) wsum[cur][warp_in][k] = a[k];
        acc[0] = acc[1] = acc[2] = 0.0;
    };
    if constexpr (!kPrimeEarly) ring_prime<XRing::NSTAGE>(n_tiles, warp, n_warps, issue);
    ring_run<XRing::NSTAGE>(n_tiles, warp, n_warps, issue, [&](int64_t t, int s) {
        seek(cb, (int32_t)t);
        if (cb.c != cur) {                                         // warp-uniform: the tile is the warp's
            if (cur >= 0) flush();
            cur = cb.c;
            const float4 k4 = kcs[cur];
            kc.G = k4.x;
            kc.denom = k4.y;
            kc.rdenom = k4.z;
            kc.denom_ok = k4.w != 0.0f;
        }
        uint32_t w[EPT / 2];
        ring.read(s, 0, w);
        // Every tensor of a batch shares the rotation, and none asks for the MMA scale
        // layout.  The rotated UE-scale kernels take both as compile-time facts (the
        // constant from the first entry, no layout test): measured 5% faster there.
        // The others read them per tensor, which measured 1-3% faster for them: in
        // these register-bound loops the allocation, not the instruction count,
        // decides.
        constexpr bool kShared = FMT != kE8M0 && K != 0;
        const QuantParams& q = P.t[kShared ? 0 : cur];
        quantize_unit<FMT, B, K, true, true, !kShared>(P.t[cur], (int64_t)((int32_t)t - cb.t0) * 32 + lane, w,
                                                       lane, kc, tabs[FMT == kE8M0 ? 0 : cur], nz, acc, pol,
                                                       q.c_hi, q.c_lo);
    });
    if (cur >= 0) flush();
    __syncthreads();
    // per-CTA partials of every tensor, warps summed in index order
    if (threadIdx.x < (unsigned)(P.count * 4)) {
        const int c = threadIdx.x >> 2, k = threadIdx.x & 3;
        double sum = 0.0;
        for (int w = 0; w < kWarps; ++w) sum += wsum[c][w][k];
        P.t[c].partials[(int64_t)blockIdx.x * 4 + k] = sum;
    }
    finish_partials_batch(P);
}

// ---------------------------------------------------------------- MSE-optimised block scales
// "Bridging the Gap", s3 (MR-GPTQ, MSE-optimised grids): each block's scale is
// the code of least squared reconstruction error among the max-rule code s0,
// s0+1 .. s0+above and s0-1 .. s0-below, tried in that order; codes outside the
// finite range are skipped and a candidate wins only with a strictly smaller
// error, so ties keep the earlier code.  The error of a candidate is the fp32
// sum of d^2, d = fp32(y - v), v = fp32(decode(code) S) (0 for S = 0).

// Block scale and its reciprocal for a candidate code, and whether the code is
// a finite scale of the format.  UE formats read the per-tensor table; E8M0
// scales are powers of two with exact reciprocals (2^-127 for byte 254).
template <int FMT>
__device__ __forceinline__ bool candidate_scale(int c, const float2* tab, float& S, float& R)
{
    if constexpr (FMT == kE8M0) {
        if (c < 0 || c > 254) return false;
        S = e8m0_decode((uint32_t)c);
        R = c == 254 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(254 - c) << 23);
        return true;
    } else {
        if (c < 0 || c > (FMT == kUE4M3 ? 0x7e : 0xfe)) return false;
        const float2 e = tab[c];
        S = e.x;
        R = e.y;
        return true;
    }
}

template <int FMT, int B, int K>
__device__ __forceinline__ void search_unit(const QuantParams& p, int64_t u, const uint32_t (&w)[EPT / 2], int lane,
                                            const ScaleConsts& kc, const float2* tab, float nz, uint64_t pol)
{
    using S = UnitShape<B, K>;
    constexpr int NB = S::NB, BE = S::BE;
    f32x2 v[EPT / 2];
    load_unit<K>(w, v, lane, p.c_hi, p.c_lo);
    float m[NB];
    if constexpr (K == 0) block_max_words<B>(w, m);
    else block_max<B, K>(v, m);

    float s0S[NB], s0R[NB];
    uint32_t s0[NB];
    unit_scales<FMT, NB>(m, kc, tab, s0, s0S, s0R);

    uint32_t best[NB];
    float best_err[NB];
    uint32_t cw[EPT / 8];
    const f32x2 nz2 = pk(nz, nz);
    const int ncand = 1 + p.above + p.below;
    for (int j = 0; j < ncand; ++j) {
        const int delta = j == 0 ? 0 : (j <= p.above ? j : p.above - j);
        float Sc[NB], Rc[NB];
        bool ok[NB], quot_ok[NB];
#pragma unroll
        for (int bi = 0; bi < NB; ++bi) {
            ok[bi] = candidate_scale<FMT>((int)s0[bi] + delta, tab, Sc[bi], Rc[bi]);
            if (!ok[bi]) Sc[bi] = Rc[bi] = 0.0f;
            // the remainder-corrected quotient needs S in its range and |m / S| <= 2^60
            quot_ok[bi] = FMT == kE8M0 || (__fmul_rn(m[bi], Rc[bi]) <= kQuotMax);
        }
        uint32_t cj[EPT / 8];
        f32x2 bsum[NB];
#pragma unroll
        for (int bi = 0; bi < NB; ++bi) bsum[bi] = pk(0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k) {
            const int bi = (8 * k) / BE;
            const f32x2* vk = v + 4 * k;
            uint32_t h[4];
            if (Sc[bi] == 0.0f) {
                cj[k] = 0u;                                         // zero-rounded: every v is 0
#pragma unroll
                for (int q = 0; q < 4; ++q) h[q] = 0u;
            } else if (FMT == kE8M0) {
                const f32x2 r = pk(Rc[bi], Rc[bi]);
                cj[k] = pack_pairs_dec(mul2(vk[0], r), mul2(vk[1], r), mul2(vk[2], r), mul2(vk[3], r), h);
            } else if (quot_ok[bi]) {
                const f32x2 R2 = pk(Rc[bi], Rc[bi]), nS2 = pk(-Sc[bi], -Sc[bi]);
                cj[k] = pack_pairs_dec(div2_cr(vk[0], R2, nS2), div2_cr(vk[1], R2, nS2), div2_cr(vk[2], R2, nS2),
                                       div2_cr(vk[3], R2, nS2), h);
            } else {
                cj[k] = pack_pairs_div(vk[0], vk[1], vk[2], vk[3], Sc[bi]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t hh;
                    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
                        : "=r"(hh) : "r"((cj[k] >> (8 * q)) & 0xffu));
                    h[q] = hh;
                }
            }
            const f32x2 s2 = pk(Sc[bi], Sc[bi]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                __half2 hh = *reinterpret_cast<__half2*>(&h[q]);
                const f32x2 g = pk(__low2float(hh), __high2float(hh));
                const f32x2 d = sub2(vk[q], fma2(g, s2, nz2));        // y - fp32(g S)
                bsum[bi] = fma2(d, d, bsum[bi]);
            }
        }
#pragma unroll
        for (int bi = 0; bi < NB; ++bi) {
            float se, so;
            upk(bsum[bi], se, so);
            float e = __fadd_rn(se, so);
            if constexpr (S::LPB > 1) e = group_sum<S::LPB>(e);
            const bool take = j == 0 || (ok[bi] && e < best_err[bi]);
            if (take) {
                best_err[bi] = e;
                best[bi] = (uint32_t)((int)s0[bi] + delta);
#pragma unroll
                for (int k = 0; k < EPT / 8; ++k)
                    if ((8 * k) / BE == bi) cw[k] = cj[k];
            }
        }
    }
    store_unit<B, K, false>(p, u, cw, best, lane, pol);
}

template <int FMT, int B, int K>
__global__ void __launch_bounds__(kThreads, 2) search_kernel(QuantParams p)
{
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem_ring[];
    const int lane = threadIdx.x & 31;
    const int64_t n_tiles = (p.n + 32 * EPT - 1) / (32 * EPT);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const XRing ring = warp_ring<XRing, K>(smem_ring);

    float G = 1.0f;
    if (FMT != kE8M0 && p.gsrc != nullptr) {
        G = *p.gsrc;
        if (p.gdst != nullptr) {
            G = G > 0.0f ? __fdiv_rn(G, 2688.0f) : 1.0f;
            if (blockIdx.x == 0 && threadIdx.x == 0) *p.gdst = G;
        }
    }
    const ScaleConsts kc = scale_consts(G);
    __shared__ float2 tab[256];
    if constexpr (FMT != kE8M0) fill_scale_table<FMT>(tab, G);
    __syncthreads();
    const float nz = __uint_as_float(0x80000000u | (uint32_t)((uint64_t)p.n >> 63));
    // x and the codes are read again by the MSE and dequantize passes: default L2 policy
    stream_tiles(ring, reinterpret_cast<const uint8_t*>(p.x), 2 * p.n, n_tiles, warp, n_warps, lane,
                 [&](int64_t t, int s) {
                     uint32_t w[EPT / 2];
                     ring.read(s, 0, w);
                     search_unit<FMT, B, K>(p, t * 32 + lane, w, lane, kc, tab, nz, 0);
                 });
}

// ---------------------------------------------------------------- per-tensor amax
// One launch takes the maxima of up to kAmaxBatch tensors: their ring tiles are
// numbered one after the other (tensor c owns tiles tile0[c] .. tile0[c+1]-1),
// and the warps stride over all of them, so a batch of small tensors fills the
// GPU like one large tensor.
constexpr int kAmaxBatch = 32;
constexpr int kAmaxTileElems = 32 * EPT;    // elements of one ring tile

struct AmaxParams {
    const uint16_t* x[kAmaxBatch];
    int64_t n[kAmaxBatch];                  // elements of each tensor
    int64_t tile0[kAmaxBatch + 1];          // first tile of each tensor; tile0[count] = all tiles
    unsigned int* amax_bits[kAmaxBatch];    // max |y| as fp32 bits (non-negative floats order as integers)
    int count;
    float c_hi, c_lo;                       // 1/sqrt(K) split in two fp32 parts
};

template <int K>
__global__ void __launch_bounds__(kThreads) amax_kernel(AmaxParams p)
{
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem_ring[];
    const int lane = threadIdx.x & 31;
    const int64_t n_tiles = p.tile0[p.count];
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const XRing ring = warp_ring<XRing, K>(smem_ring);
    // A warp's tiles rise, so its tensors do too: one cursor for the copies issued
    // ahead and one for the tile being reduced, each holding its tensor's tile range
    // (and source) in registers so that a tile of the same tensor costs one compare.
    // Tiles past tile0[count] are never issued, so both cursors stay below count.
    struct Cursor {
        int c;
        int64_t t0, t1;
    };
    auto seek = [&](Cursor& k, int64_t t) {
        while (t >= k.t1) {
            ++k.c;
            k.t0 = k.t1;
            k.t1 = p.tile0[k.c + 1];
        }
    };
    Cursor ci{0, 0, p.tile0[1]}, cb{0, 0, p.tile0[1]};
    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.x[0]);
    int64_t nbytes = 2 * p.n[0];
    int src_c = 0, cur = -1;
    float mx = 0.0f;
    uint32_t mb = 0;                                       // two halves whose magnitudes are the largest seen
    auto flush = [&]() {
        float m;
        if constexpr (K == 0) {
            m = bf16x2_absmax_f32(mb);
        } else {
            // y = fp32(s c_hi + fp32(s c_lo)) rounds monotonically and symmetrically in s
            // (c_lo = 0 for K = 16), so the largest |y| is the normalised largest |s|: the
            // quantizer's own maxima exactly
            m = __fmaf_rn(mx, p.c_hi, __fmul_rn(mx, p.c_lo));
        }
        m = group_max<32>(m);
        if (lane == 0 && m > 0.0f) atomicMax(p.amax_bits[cur], __float_as_uint(m));
        mx = 0.0f;
        mb = 0;
    };
    stream_tiles_with<XRing::NSTAGE>(
        n_tiles, warp, n_warps,
        [&](int64_t t, int s) {
            seek(ci, t);
            if (ci.c != src_c) {
                src_c = ci.c;
                src = reinterpret_cast<const uint8_t*>(p.x[src_c]);
                nbytes = 2 * p.n[src_c];
            }
            ring.issue(src, nbytes, (t - ci.t0) * XRing::TILE_BYTES, s, lane);
        },
        [&](int64_t t, int s) {
            seek(cb, t);
            if (cb.c != cur) {                              // warp-uniform: the tile is the warp's
                if (cur >= 0) flush();
                cur = cb.c;
            }
            uint32_t w[EPT / 2];
            ring.read(s, 0, w);
            if constexpr (K == 0) {
                // packed bf16 maxima of magnitudes (finite inputs: the largest magnitude's
                // pattern; the sign bits are meaningless and masked at the flush)
#pragma unroll
                for (int k = 0; k < EPT / 2; ++k) mb = bf16x2_absmax(mb, w[k]);
            } else {
                // the raw Sylvester sums (magnitudes only: their signs do not
                // matter); 1/sqrt(K) is applied once, to the maximum
                f32x2 v[EPT / 2];
                unit_sums<K>(w, v, lane);
                mx = fmaxf(mx, pairs_absmax<EPT>(v));
            }
        });
    if (cur >= 0) flush();
}

// Zero the amax slots of a batch (before a batch that overwrites them).
static __global__ void amax_zero_kernel(AmaxParams p)
{
    if ((int)threadIdx.x < p.count) *p.amax_bits[threadIdx.x] = 0u;
}

// G = amax / (6 * 448) (correctly rounded), or 1 for an all-zero tensor.
static __global__ void global_scale_kernel(const float* amax_in, float* gscale)
{
    const float amax = *amax_in;
    *gscale = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// Block scale from its code (decoded; G applied for the UE formats).
__device__ __forceinline__ float decode_scale(uint32_t c, int fmt, float G)
{
    if (fmt == kE8M0) return e8m0_decode(c);
    if (fmt == kUE4M3) return __fmul_rn(ue4m3_decode(c), G);
    return __fmul_rn(ue5m3_decode(c), G);
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

// A lane owns DPL = 128 consecutive elements per tile: their 64 code bytes
// stream through the ring, their DPL/B scale bytes are one vector load fetched
// a tile ahead, and a rotation run of up to 128 elements stays in registers.
constexpr int DPL = 128;

template <int B>
struct DeqScales {
    static constexpr int NSB = B <= DPL ? DPL / B : 1;            // scale bytes per lane per tile
    static constexpr int LPB = B <= DPL ? 1 : B / DPL;            // lanes per block
};

template <int B>
__device__ __forceinline__ void fetch_scale_bytes(const uint8_t* __restrict__ scales, int64_t n, int64_t e0,
                                                  uint32_t (&c)[DeqScales<B>::NSB])
{
    constexpr int NSB = DeqScales<B>::NSB;
    const int64_t nblk = n / B;
    const int64_t b0 = e0 / B;
    if constexpr (NSB >= 4) {
        if (b0 + NSB <= nblk) {
            if constexpr (NSB == 4) {
                const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(scales + b0));
#pragma unroll
                for (int i = 0; i < 4; ++i) c[i] = (v >> (8 * i)) & 0xffu;
            } else if constexpr (NSB == 8) {
                const uint2 v = __ldg(reinterpret_cast<const uint2*>(scales + b0));
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    c[i] = (v.x >> (8 * i)) & 0xffu;
                    c[4 + i] = (v.y >> (8 * i)) & 0xffu;
                }
            } else {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(scales + b0));
                const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < NSB; ++i) c[i] = (vv[i / 4] >> (8 * (i % 4))) & 0xffu;
            }
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < NSB; ++i) c[i] = (b0 + i < nblk) ? (uint32_t)__ldg(scales + b0 + i) : 0u;
}

template <int B, int K, bool F32OUT>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(DequantParams p)
{
    pdl_wait();
    pdl_release();
    const uint64_t pol = l2_evict_first();        // outputs: not read again in the step
    constexpr int NSB = DeqScales<B>::NSB;
    constexpr int EPB = B <= DPL ? B : DPL;                       // elements of a block in a lane
    using R = Ring<64, 1>;                                        // 64 code bytes per lane per tile
    extern __shared__ __align__(128) uint8_t smem_ring[];
    const int lane = threadIdx.x & 31;
    const int64_t n_tiles = (p.n + 32 * DPL - 1) / (32 * DPL);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const R ring = warp_ring<R>(smem_ring);
    const float G = (p.fmt != kE8M0 && p.gsrc != nullptr) ? *p.gsrc : 1.0f;

    uint32_t sc_next[NSB];
    if (warp < n_tiles) fetch_scale_bytes<B>(p.scales, p.n, (warp * 32 + lane) * DPL, sc_next);

    stream_tiles(ring, p.codes, p.n / 2, n_tiles, warp, n_warps, lane, [&](int64_t t, int s) {
        const int64_t e0 = (t * 32 + lane) * DPL;
        uint32_t scb[NSB];
#pragma unroll
        for (int i = 0; i < NSB; ++i) scb[i] = sc_next[i];
        if (t + n_warps < n_tiles) fetch_scale_bytes<B>(p.scales, p.n, ((t + n_warps) * 32 + lane) * DPL, sc_next);
        uint32_t cw[16];
        ring.read(s, 0, cw);
        if (e0 >= p.n) return;
        // chunks of CH elements: decode, rotate back (one run), round, store
        constexpr int CH = K == 0 ? 16 : K;
#pragma unroll
        for (int c0 = 0; c0 < DPL; c0 += CH) {
            f32x2 v[CH / 2];
#pragma unroll
            for (int k = 0; k < CH / 8; ++k) {
                const int kk = c0 / 8 + k;                             // code word index in the lane's 128
                f32x2 g[4];
                decode8(cw[kk], g);
                const float sv = decode_scale(scb[(8 * kk) / EPB], p.fmt, G);
                const f32x2 s2 = pk(sv, sv);
#pragma unroll
                for (int j = 0; j < 4; ++j) v[4 * k + j] = K > 0 ? mul2_rounded(g[j], s2) : mul2(g[j], s2);
            }
            if constexpr (K > 0) {
                fwht_inreg<CH, K>(v);
                normalize<CH>(v, p.c_hi, p.c_lo);
            }
            const int64_t ec = e0 + c0;
            const bool full = ec + CH <= p.n;
            if constexpr (F32OUT) {
                float* dst = reinterpret_cast<float*>(p.y) + ec;
                if (full) {
#pragma unroll
                    for (int k = 0; k < CH / 8; ++k) {
                        float a[8];
                        upk(v[4 * k], a[0], a[1]);
                        upk(v[4 * k + 1], a[2], a[3]);
                        upk(v[4 * k + 2], a[4], a[5]);
                        upk(v[4 * k + 3], a[6], a[7]);
                        stg256(dst + 8 * k, __float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                               __float_as_uint(a[3]), __float_as_uint(a[4]), __float_as_uint(a[5]),
                               __float_as_uint(a[6]), __float_as_uint(a[7]), pol);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < CH / 2; ++k) {
                        float a, b;
                        upk(v[k], a, b);
                        if (ec + 2 * k < p.n) {
                            dst[2 * k] = a;
                            dst[2 * k + 1] = b;
                        }
                    }
                }
            } else {
                uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(p.y) + ec);
#pragma unroll
                for (int k = 0; k < CH / 16; ++k) {
                    uint32_t o[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float a, b;
                        upk(v[8 * k + j], a, b);
                        __nv_bfloat162 hb = __floats2bfloat162_rn(a, b);
                        o[j] = *reinterpret_cast<uint32_t*>(&hb);
                    }
                    if (full) {
                        stg256(dst + 8 * k, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7], pol);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (ec + 16 * k + 2 * j < p.n) dst[8 * k + j] = o[j];
                    }
                }
            }
        }
    });
}

// ---------------------------------------------------------------- dequantize, interleaved chunks
// For rotation runs of at most 16 elements.  A warp's tile is 32 x 8 chunks
// of 16 elements; chunk c of lane l holds elements tile + (32 c + l) * 16 ..
// + 15, so each store instruction of the warp writes 32 consecutive chunks
// (1 KiB of bf16, 2 KiB of fp32) and every lane's loads and stores are full
// 32-byte sectors.  A ring stage holds the tile's 2 KiB of codes followed by
// its scale bytes (4096 / B, at least one 16-byte chunk), copied with 16-byte
// cp.async; the block scales come from a per-tensor table of the 256 codes.
constexpr int kDqChunk = 16;
constexpr int kDqCpt = 8;                                    // chunks per lane per tile
constexpr int kDqTile = 32 * kDqCpt * kDqChunk;              // 4096 elements

template <int B>
struct DqStage {
    static constexpr int CODE_BYTES = kDqTile / 2;
    static constexpr int SC_RAW = kDqTile / B;               // 16 .. 512 scale bytes per tile
    static constexpr int SC_BYTES = SC_RAW < 16 ? 16 : SC_RAW;
    static constexpr int SC_CHUNKS = SC_BYTES / 16;          // 1 .. 32
    static constexpr int BYTES = CODE_BYTES + SC_BYTES;
    static constexpr int NSTAGE = kRingBytesPerWarp / BYTES;
    static_assert(NSTAGE >= 2 && SC_CHUNKS <= 32, "stage layout");
};

// Copies of tile t into stage s (sb: its shared address); bytes past the end
// of the codes or scales are zero-filled and never read from global memory.
template <int B>
__device__ __forceinline__ void dq_issue(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                         int64_t code_bytes, int64_t scale_bytes, int64_t t, uint32_t sb, int lane)
{
    using D = DqStage<B>;
    const int64_t co = t * (int64_t)D::CODE_BYTES, so = t * (int64_t)D::SC_RAW;
    if (co + D::CODE_BYTES <= code_bytes && so + D::SC_BYTES <= scale_bytes) {
#pragma unroll
        for (int j = 0; j < D::CODE_BYTES / 512; ++j)
            cp_async16(sb + 16u * (uint32_t)(lane + 32 * j), codes + co + 16 * (lane + 32 * j), 16u);
        if (lane < D::SC_CHUNKS) cp_async16(sb + D::CODE_BYTES + 16u * lane, scales + so + 16 * lane, 16u);
    } else {
#pragma unroll
        for (int j = 0; j < D::CODE_BYTES / 512; ++j) {
            const int64_t o = co + 16 * (lane + 32 * j), left = code_bytes - o;
            const uint32_t cnt = left >= 16 ? 16u : (left > 0 ? (uint32_t)left : 0u);
            cp_async16(sb + 16u * (uint32_t)(lane + 32 * j), cnt ? (const void*)(codes + o) : (const void*)codes, cnt);
        }
        if (lane < D::SC_CHUNKS) {
            const int64_t o = so + 16 * lane, left = scale_bytes - o;
            const uint32_t cnt = left >= 16 ? 16u : (left > 0 ? (uint32_t)left : 0u);
            cp_async16(sb + D::CODE_BYTES + 16u * lane, cnt ? (const void*)(scales + o) : (const void*)scales, cnt);
        }
    }
}

__device__ __forceinline__ uint2 lds64(uint32_t smem_addr)
{
    uint2 r;
    asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(smem_addr));
    return r;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t smem_addr)
{
    uint32_t r;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(r) : "r"(smem_addr));
    return r;
}

template <int B, int K, bool F32OUT>
__global__ void __launch_bounds__(kThreads) dequantize_il_kernel(DequantParams p)
{
    static_assert(K == 0 || K == kDqChunk, "interleaved chunks hold rotation runs of at most 16");
    pdl_wait();
    pdl_release();
    const uint64_t pol = l2_evict_first();        // outputs: not read again in the step
    using D = DqStage<B>;
    extern __shared__ __align__(128) uint8_t smem_ring[];
    __shared__ float tab[256];                                   // block scale by code
    const int lane = threadIdx.x & 31;
    const float G = (p.fmt != kE8M0 && p.gsrc != nullptr) ? *p.gsrc : 1.0f;
    for (int c = threadIdx.x; c < 256; c += kThreads) tab[c] = decode_scale((uint32_t)c, p.fmt, G);
    __syncthreads();

    const int64_t n_tiles = (p.n + kDqTile - 1) / kDqTile;
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const uint32_t ring = (uint32_t)__cvta_generic_to_shared(smem_ring) + (uint32_t)((threadIdx.x >> 5) * kRingBytesPerWarp);
    const int64_t code_bytes = p.n / 2, scale_bytes = p.n / B;
    constexpr int NS = D::NSTAGE;

    int64_t t_issue = warp;
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) {
        if (t_issue < n_tiles) dq_issue<B>(p.codes, p.scales, code_bytes, scale_bytes, t_issue, ring + s * D::BYTES, lane);
        cp_async_commit();
        t_issue += n_warps;
    }
    int stage = 0;
    for (int64_t t = warp; t < n_tiles; t += n_warps) {
        const int s_new = stage == 0 ? NS - 1 : stage - 1;
        if (t_issue < n_tiles) dq_issue<B>(p.codes, p.scales, code_bytes, scale_bytes, t_issue, ring + s_new * D::BYTES, lane);
        cp_async_commit();
        t_issue += n_warps;
        cp_async_wait<NS - 1>();
        __syncwarp();
        const uint32_t sb = ring + stage * D::BYTES;
        const int64_t tile0 = t * kDqTile;
#pragma unroll 2
        for (int c = 0; c < kDqCpt; ++c) {
            const int ch = 32 * c + lane;                        // chunk index in the tile
            const int64_t e0 = tile0 + (int64_t)ch * kDqChunk;
            if (e0 >= p.n) break;
            const uint2 cw = lds64(sb + 8u * (uint32_t)ch);
            float s0, s1;
            if constexpr (B == 8) {
                s0 = tab[lds_u8(sb + D::CODE_BYTES + 2u * ch)];
                s1 = tab[lds_u8(sb + D::CODE_BYTES + 2u * ch + 1u)];
            } else {
                const uint32_t sc = lds_u8(sb + D::CODE_BYTES + (uint32_t)((ch * kDqChunk) / B));
                s0 = s1 = tab[sc];
            }
            f32x2 g[8], v[8];
            decode8(cw.x, *reinterpret_cast<f32x2(*)[4]>(&g[0]));
            decode8(cw.y, *reinterpret_cast<f32x2(*)[4]>(&g[4]));
            const f32x2 S0 = pk(s0, s0), S1 = pk(s1, s1);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = K > 0 ? mul2_rounded(g[j], j < 4 ? S0 : S1) : mul2(g[j], j < 4 ? S0 : S1);
            if constexpr (K > 0) {
                fwht_inreg<kDqChunk, K>(v);
                normalize<kDqChunk>(v, p.c_hi, p.c_lo);
            }
            const bool full = e0 + kDqChunk <= p.n;
            if constexpr (F32OUT) {
                float* dst = reinterpret_cast<float*>(p.y) + e0;
                float a[16];
#pragma unroll
                for (int j = 0; j < 8; ++j) upk(v[j], a[2 * j], a[2 * j + 1]);
                if (full) {
                    stg256(dst, __float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]), __float_as_uint(a[3]),
                           __float_as_uint(a[4]), __float_as_uint(a[5]), __float_as_uint(a[6]), __float_as_uint(a[7]), pol);
                    stg256(dst + 8, __float_as_uint(a[8]), __float_as_uint(a[9]), __float_as_uint(a[10]),
                           __float_as_uint(a[11]), __float_as_uint(a[12]), __float_as_uint(a[13]), __float_as_uint(a[14]),
                           __float_as_uint(a[15]), pol);
                } else {
                    for (int j = 0; j < kDqChunk; ++j)
                        if (e0 + j < p.n) dst[j] = a[j];
                }
            } else {
                uint32_t o[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float a, b;
                    upk(v[j], a, b);
                    __nv_bfloat162 hb = __floats2bfloat162_rn(a, b);
                    o[j] = *reinterpret_cast<uint32_t*>(&hb);
                }
                uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(p.y) + e0);
                if (full) {
                    stg256(dst, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7], pol);
                } else {
                    for (int j = 0; j < 8; ++j)
                        if (e0 + 2 * j < p.n) dst[j] = o[j];
                }
            }
        }
        stage = stage + 1 == NS ? 0 : stage + 1;
        __syncwarp();
    }
    cp_async_wait_all();
}

// ---------------------------------------------------------------- block MSE of given codes
struct MseParams {
    const uint16_t* x;
    const uint8_t* codes;
    const uint8_t* scales;
    const float* gsrc;
    int64_t n;
    int fmt;
    float* block_mse;      // n/B floats or nullptr
    double* partials;      // [gridDim.x][4]
    unsigned int* done;    // completion counter (0 at launch, left 0)
    double* terms;         // the four tensor terms
    float c_hi, c_lo;
};

template <int N>
__device__ __forceinline__ float tree_sum(const float* a)
{
    if constexpr (N == 1) return a[0];
    else return __fadd_rn(tree_sum<N / 2>(a), tree_sum<N / 2>(a + N / 2));
}

// Codes and scale bytes of a unit (zeros past the end).
template <int B, int K>
__device__ __forceinline__ void load_unit_codes(const uint8_t* __restrict__ codes,
                                                const uint8_t* __restrict__ scales, int64_t n, int64_t u,
                                                uint32_t (&cw)[EPT / 8], uint32_t (&sb)[UnitShape<B, K>::NB])
{
    using S = UnitShape<B, K>;
    const int64_t e0 = u * EPT;
    if (e0 + EPT <= n) {
        const uint4 r = __ldg(reinterpret_cast<const uint4*>(codes + e0 / 2));
        cw[0] = r.x;
        cw[1] = r.y;
        cw[2] = r.z;
        cw[3] = r.w;
    } else {
        const int64_t nbytes = e0 < n ? (n - e0) / 2 : 0;
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (4 * k + j < nbytes) word |= (uint32_t)codes[e0 / 2 + 4 * k + j] << (8 * j);
            cw[k] = word;
        }
    }
#pragma unroll
    for (int bi = 0; bi < S::NB; ++bi) {
        const int64_t e = e0 + (int64_t)bi * S::BE;
        sb[bi] = e < n ? (uint32_t)__ldg(scales + e / B) : 0u;
    }
}

// The codes may come from anywhere, so the block maximum's error is taken at
// the first element of largest |y| (the oracle's reading), not from the
// largest dequantized value.
template <int B, int K>
__global__ void __launch_bounds__(kThreads) block_mse_kernel(MseParams p)
{
    pdl_wait();
    pdl_release();
    using S = UnitShape<B, K>;
    constexpr int NB = S::NB, BE = S::BE, LPB = S::LPB;
    extern __shared__ __align__(128) uint8_t smem_ring[];
    const int lane = threadIdx.x & 31;
    const int64_t n_tiles = (p.n + 32 * EPT - 1) / (32 * EPT);
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const XRing ring = warp_ring<XRing, K>(smem_ring);
    const float G = (p.fmt != kE8M0 && p.gsrc != nullptr) ? *p.gsrc : 1.0f;

    double acc_total = 0.0, acc_nonmax = 0.0, acc_max = 0.0, acc_zero = 0.0;
    // codes and scales of the next tile are fetched one iteration ahead
    uint32_t cw_next[EPT / 8], sb_next[NB];
    if (warp < n_tiles) load_unit_codes<B, K>(p.codes, p.scales, p.n, warp * 32 + lane, cw_next, sb_next);
    stream_tiles(ring, reinterpret_cast<const uint8_t*>(p.x), 2 * p.n, n_tiles, warp, n_warps, lane,
                 [&](int64_t t, int s) {
        const int64_t u = t * 32 + lane;
        uint32_t cw[EPT / 8], sb[NB];
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k) cw[k] = cw_next[k];
#pragma unroll
        for (int bi = 0; bi < NB; ++bi) sb[bi] = sb_next[bi];
        if (t + n_warps < n_tiles) load_unit_codes<B, K>(p.codes, p.scales, p.n, (t + n_warps) * 32 + lane, cw_next, sb_next);
        uint32_t w[EPT / 2];
        ring.read(s, 0, w);
        const int64_t e0 = u * EPT;
        f32x2 yp[EPT / 2];
        load_unit<K>(w, yp, lane, p.c_hi, p.c_lo);
        float m[NB];
        block_max<B, K>(yp, m);
        float y[EPT], v[EPT];
#pragma unroll
        for (int k = 0; k < EPT / 8; ++k) {
            f32x2 g[4];
            decode8(cw[k], g);
            const int bi = (8 * k) / BE;
            const float sv = e0 + (int64_t)bi * BE < p.n ? decode_scale(sb[bi], p.fmt, G) : 0.0f;
            const f32x2 s2 = pk(sv, sv);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                upk(mul2_rounded(g[j], s2), v[8 * k + 2 * j], v[8 * k + 2 * j + 1]);
                upk(yp[4 * k + j], y[8 * k + 2 * j], y[8 * k + 2 * j + 1]);
            }
        }
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
            for (int i = 0; i < BE; ++i)
                if (i == first) emax = e2[i];
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
                if (p.block_mse) p.block_mse[eb / B] = __fmul_rn(bsum, 1.0f / (float)B);
                acc_total += (double)bsum;
                if (vmax == 0.0f) acc_zero += (double)bsum;
                else {
                    acc_nonmax += (double)nonmax;
                    acc_max += (double)bmax;
                }
            }
        }
    });
    cta_partials(acc_total, acc_nonmax, acc_max, acc_zero, p.partials);
    finish_partials(p.partials, p.done, p.n, p.terms);
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

// Scale codes one value at a time through the quantizer's own encoders: UE
// formats give the code nearest to s (the quantizer applies the same encoder,
// two values at a time for UE4M3, to the correctly rounded m / fp32(6G)),
// E8M0 the byte of a block whose maximum is s.
static __global__ void __launch_bounds__(kThreads) scale_encode_kernel(const float* __restrict__ s, int64_t n,
                                                                      int fmt, uint8_t* __restrict__ out)
{
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = 2 * ((int64_t)blockIdx.x * kThreads + threadIdx.x); i < n; i += 2 * stride) {
        const float s0 = s[i], s1 = (i + 1 < n) ? s[i + 1] : 0.0f;
        uint32_t c0, c1;
        if (fmt == kE8M0) {
            c0 = e8m0_from_amax(s0);
            c1 = e8m0_from_amax(s1);
        } else if (fmt == kUE4M3) {
            const uint32_t cc = ue4m3_encode2(s0, s1);
            c0 = cc & 0xffu;
            c1 = cc >> 8;
        } else {
            c0 = ue5m3_encode(s0);
            c1 = ue5m3_encode(s1);
        }
        out[i] = (uint8_t)c0;
        if (i + 1 < n) out[i + 1] = (uint8_t)c1;
    }
}

}  // namespace fp4q
