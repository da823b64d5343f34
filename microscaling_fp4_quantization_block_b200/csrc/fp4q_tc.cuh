// fp4q_tc.cuh -- the block-wise Hadamard rotation on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory), feeding the quantizer.
//
// "Bridging the Gap", s3.1/s3.4: the online rotation is a block-diagonal
// Hadamard transform fused with quantization and scale computation.  For a
// rotation of K = 16 or 32 consecutive elements the input is viewed as rows of
// KR = 32 elements (one or two rotation runs per row) and rotated as one GEMM
// per tile of 128 rows:
//
//     D[m][n] = sum_k A[m][k] B[n][k],   A = x (bf16, 128 x 32),
//                                        B = I_{32/K} (x) H_K  (bf16 +-1 / 0),
//
// with fp32 accumulators in tensor memory (TMEM).  Every product is exact (a
// bf16 value times +-1) and only the accumulation rounds; the result is then
// scaled by 1/sqrt(K) exactly as the butterfly path scales it.  Row m of D
// lands in TMEM lane m, so after one tcgen05.ld each thread of a warpgroup
// holds the 32 rotated values of "its" row: the same 32-element unit the
// quantizer works on, with no shuffles.
//
// Pipeline (per warpgroup of 128 threads, independent of the other warpgroup
// of the CTA): a ring of NSTAGE tiles in shared memory filled by 16-byte
// cp.async copies straight into the 64-byte-swizzled K-major layout the MMA
// reads; one thread issues the two K=16 MMAs of tile i+1 into one of two TMEM
// buffers while all threads read and quantize tile i from the other.  MMA
// completion is tracked by tcgen05.commit on an mbarrier; every wait on it is
// bounded and, when the bound runs out, records a fault (fp4q_device_fault)
// and stops the warpgroup's work without hanging.
#pragma once

#include "fp4q_kernels.cuh"

namespace fp4q {
namespace tc {

constexpr int KR = 32;                          // elements per MMA row
constexpr int ROWS = 128;                       // rows per tile (M of the MMA), one per thread of a warpgroup
constexpr int TILE_ELEMS = ROWS * KR;           // 4096
constexpr int STAGE_BYTES = ROWS * KR * 2;      // 8 KiB of bf16
constexpr int NSTAGE = 4;                       // ring stages per warpgroup
constexpr int WGS = kThreads / 128;             // warpgroups per CTA (2)
constexpr int TMEM_COLS_WG = 2 * KR;            // two fp32 accumulator buffers of 32 columns
constexpr int TMEM_COLS = WGS * TMEM_COLS_WG;   // 128 (a power of two >= 32)
constexpr int B_BYTES = KR * KR * 2;            // the rotation matrix, 2 KiB
// dynamic shared memory: 1 KiB of slack to align the swizzled buffers to 1 KiB,
// the rotation matrix, the rings, then mbarriers and the TMEM address slot
constexpr int SMEM_BYTES = 1024 + B_BYTES + WGS * NSTAGE * STAGE_BYTES + 64;

// Instruction descriptor of tcgen05.mma kind::f16: D fp32 (bits 4-5 = 1),
// A and B bf16 (bits 7-9, 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdescBf16F32 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(KR >> 3) << 17) |
                                   ((uint32_t)(ROWS >> 4) << 24);

// Shared-memory matrix descriptor of a K-major operand in the 64-byte swizzle
// layout (rows of 64 bytes, 8-row groups 512 bytes apart): start address >> 4
// in bits 0-13, leading offset 1 (unused for swizzled K-major) in bits 16-29,
// stride offset 512 >> 4 in bits 32-45, version 1 in bits 46-47, layout type 4
// (SWIZZLE_64B) in bits 61-63.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t smem_addr)
{
    return (uint64_t)((smem_addr >> 4) & 0x3fffu) | ((uint64_t)1u << 16) | ((uint64_t)(512u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)4u << 61);
}

// Byte offset of 16-byte chunk j (0..3) of row r in the 64-byte swizzle layout:
// the chunk index is XORed with bits 1-2 of the row (address bits 7-8).
__device__ __forceinline__ uint32_t sw64_offset(int r, int j)
{
    return (uint32_t)(r * 64 + 16 * (j ^ ((r >> 1) & 3)));
}

// ---------------------------------------------------------------- tcgen05 / mbarrier primitives
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// One bounded probe of the barrier's phase `parity`; true once it has completed.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Make this thread's completed generic-proxy writes to shared memory (cp.async
// data, st.shared) visible to the async proxy that the MMA reads through.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[desc_a] * B[desc_b]^T; accumulate = false overwrites D.
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t desc_a, uint64_t desc_b, uint32_t idesc,
                                         bool accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(tmem_d), "l"(desc_a), "l"(desc_b), "r"(idesc), "r"((uint32_t)accumulate)
                 : "memory");
}

// Arrive once on the mbarrier when every tcgen05 operation this thread has
// issued so far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (32x32b shape: warp w
// of a warpgroup reads lanes 32 (w % 4) .. + 31, thread l lane 32 (w % 4) + l).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
                   "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
                   "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr)
                 : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Barrier over the 128 threads of warpgroup wg (named barriers 1 and 2).
__device__ __forceinline__ void wg_sync(int wg) { asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory"); }

// Polls of an mbarrier before a wait gives up (each poll is a hardware-bounded
// try_wait; together they span far more than any MMA of this kernel takes).
constexpr uint32_t kMaxPolls = 1u << 22;

// ---------------------------------------------------------------- the rotation matrix
// B[n][k] for a rotation of K (16 or 32) on rows of 32: Sylvester H_K
// (H[i][j] = (-1)^popcount(i & j)) on the diagonal blocks, 0 elsewhere; bf16
// +1 = 0x3F80, -1 = 0xBF80.  Written in the 64-byte swizzle layout.
template <int K>
__device__ __forceinline__ void fill_rotation_matrix(uint32_t b_smem)
{
    for (int idx = threadIdx.x; idx < KR * KR / 2; idx += blockDim.x) {
        const int n = idx / (KR / 2), k = 2 * (idx % (KR / 2));
        uint32_t w = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int kk = k + h;
            uint32_t v = 0;
            if ((n / K) == (kk / K)) v = (__popc((n % K) & (kk % K)) & 1) ? 0xBF80u : 0x3F80u;
            w |= v << (16 * h);
        }
        const uint32_t off = sw64_offset(n, (2 * k) / 16) + (uint32_t)((2 * k) % 16);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(b_smem + off), "r"(w) : "memory");
    }
}

// ---------------------------------------------------------------- the pipeline
// Every tile of 4096 elements of x (bf16, n elements, n a multiple of 32) is
// rotated by the tensor cores; body(u, v) is then called by every thread for
// unit u (32 consecutive elements, index u = tile * 128 + row) with the
// rotated, not yet normalised, values v.  Rows at or past n hold zeros.
// Warpgroups walk tiles in a grid-stride loop (the same trip count for every
// thread of a warpgroup).  Returns false when an MMA wait gave up.
template <int K, typename Body>
__device__ __forceinline__ bool rotate_tiles(const uint16_t* __restrict__ x, int64_t n, uint8_t* smem_raw,
                                             unsigned int* fault, Body&& body, bool ef, uint64_t pol)
{
    const uint32_t raw = (uint32_t)__cvta_generic_to_shared(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;               // swizzle atoms need 1 KiB alignment
    const uint32_t b_smem = base;
    const int wg = threadIdx.x >> 7;
    const int t128 = threadIdx.x & 127;
    const int warp_in_wg = t128 >> 5, lane = threadIdx.x & 31;
    const uint32_t ring = base + B_BYTES + (uint32_t)(wg * NSTAGE * STAGE_BYTES);
    const uint32_t bars = base + B_BYTES + (uint32_t)(WGS * NSTAGE * STAGE_BYTES);     // 2 per warpgroup
    const uint32_t bar0 = bars + 16u * (uint32_t)wg;
    const uint32_t slot = bars + 16u * WGS;                                         // TMEM base address
    __shared__ int abort_flag[WGS];

    fill_rotation_matrix<K>(b_smem);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * WGS; ++i) mbar_init(bars + 8u * (uint32_t)i, 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (t128 == 0) abort_flag[wg] = 0;
    if (threadIdx.x < 32) tmem_alloc(slot, TMEM_COLS);
    fence_proxy_async_smem();                                    // the rotation matrix, for the MMA
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t tmem_base;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem_base) : "r"(slot) : "memory");
    const uint32_t tmem_wg = tmem_base + (uint32_t)(wg * TMEM_COLS_WG);
    const uint32_t tmem_lane = (uint32_t)(32 * warp_in_wg) << 16;

    // this thread's 4 copies of a tile: chunk g = 32 c + lane of its warp's 2 KiB
    uint32_t s_off[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int g = 32 * c + lane;
        s_off[c] = sw64_offset(32 * warp_in_wg + (g >> 2), g & 3);
    }
    const int64_t nbytes = 2 * n;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(x);
    auto issue = [&](int64_t tile, int stage) {
        const uint32_t sb = ring + (uint32_t)(stage * STAGE_BYTES);
        const int64_t off0 = tile * (int64_t)STAGE_BYTES + 2048 * warp_in_wg + 16 * lane;
        if (off0 - 16 * lane + 2048 <= nbytes) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (ef) cp_async16(sb + s_off[c], src + off0 + 512 * c, 16u, pol);
                else cp_async16(sb + s_off[c], src + off0 + 512 * c, 16u);
            }
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int64_t o = off0 + 512 * c;
                const int64_t left = nbytes - o;
                const uint32_t cnt = left >= 16 ? 16u : (left > 0 ? (uint32_t)left : 0u);
                cp_async16(sb + s_off[c], cnt ? (const void*)(src + o) : (const void*)src, cnt);
            }
        }
    };

    const int64_t n_tiles = (n + TILE_ELEMS - 1) / TILE_ELEMS;
    const int64_t first = (int64_t)blockIdx.x * WGS + wg;
    const int64_t stride = (int64_t)gridDim.x * WGS;
    const bool leader = t128 == 0;
    bool ok = true;

    auto issue_mma = [&](int stage, int buf) {
        const uint32_t a = ring + (uint32_t)(stage * STAGE_BYTES);
        const uint32_t d = tmem_wg + (uint32_t)(buf * KR);
        tc_fence_after();
        mma_bf16(d, sw64_desc(a), sw64_desc(b_smem), kIdescBf16F32, false);
        mma_bf16(d, sw64_desc(a + 32u), sw64_desc(b_smem + 32u), kIdescBf16F32, true);
        mma_commit(bar0 + 8u * (uint32_t)buf);
    };

    // prologue: NSTAGE - 1 tiles in flight, then the MMA of the first one
#pragma unroll
    for (int s = 0; s < NSTAGE - 1; ++s) {
        const int64_t t = first + s * stride;
        if (t < n_tiles) issue(t, s);
        cp_async_commit();
    }
    if (first < n_tiles) {
        cp_async_wait<NSTAGE - 2>();
        fence_proxy_async_smem();
        wg_sync(wg);
        if (leader) issue_mma(0, 0);
    }
    int64_t i = 0;
    for (int64_t t = first; t < n_tiles; t += stride, ++i) {
        // refill the stage tile i - 1 used (its MMA has completed: waited below)
        const int64_t t_fill = t + (NSTAGE - 1) * stride;
        if (t_fill < n_tiles) issue(t_fill, (int)((i + NSTAGE - 1) % NSTAGE));
        cp_async_commit();
        // the MMA of tile i + 1, once every thread's copies of it have landed and
        // every thread has read TMEM buffer (i + 1) % 2 (tile i - 1)
        cp_async_wait<NSTAGE - 2>();
        fence_proxy_async_smem();
        tc_fence_before();
        wg_sync(wg);
        const bool go = ok && abort_flag[wg] == 0;         // one shared load per warp: warp-uniform
        if (leader && go && t + stride < n_tiles) issue_mma((int)((i + 1) % NSTAGE), (int)((i + 1) & 1));
        // tile i: wait (bounded) for its MMA, then read this thread's row; the
        // decision is made per warp, since tcgen05.ld needs the whole warp
        bool have = false;
        if (go) {
            const uint32_t bar = bar0 + 8u * (uint32_t)(i & 1);
            const uint32_t parity = (uint32_t)((i >> 1) & 1);
            bool done = mbar_try_wait(bar, parity);
            for (uint32_t polls = 1; !done && polls < kMaxPolls; ++polls) done = mbar_try_wait(bar, parity);
            have = __all_sync(0xffffffffu, done);
            if (!have) {
                ok = false;
                if (lane == 0) {
                    atomicExch(fault, 1u);
                    abort_flag[wg] = 1;
                }
            }
        }
        if (have) {
            tc_fence_after();
            uint32_t r[32];
            tmem_ld32(tmem_wg + tmem_lane + (uint32_t)((i & 1) * KR), r);
            f32x2 v[EPT / 2];
#pragma unroll
            for (int k = 0; k < EPT / 2; ++k) v[k] = pk(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
            body(t * ROWS + t128, v);
        }
    }
    cp_async_wait_all();
    // every MMA this warpgroup issued has completed (each was waited on, or the
    // warpgroup gave up), so TMEM can be released
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
    return ok;
}

}  // namespace tc

// ---------------------------------------------------------------- kernels on the tensor-core rotation
// Quantize (+ fused MSE / dequantized output) with the rotation (K = 16, 32)
// on the tensor cores; outputs identical in layout to quantize_kernel's.
template <int FMT, int B, int K, bool MSE, bool DQ>
__global__ void __launch_bounds__(kThreads, 2) quantize_tc_kernel(QuantParams p)
{
    static_assert(K == 16 || K == 32, "tensor-core rotation of 16 or 32");
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem_tc[];
    const int lane = threadIdx.x & 31;

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
    // (the pipeline's first __syncthreads orders the table before any use)
    const float nz = __uint_as_float(0x80000000u | (uint32_t)((uint64_t)p.n >> 63));
    double acc[3] = {0.0, 0.0, 0.0};
    const uint64_t pol = l2_evict_first();
    tc::rotate_tiles<K>(
        p.x, p.n, smem_tc, p.fault,
        [&](int64_t u, f32x2 (&v)[EPT / 2]) {
            normalize<EPT>(v, p.c_hi, p.c_lo);
            float m[UnitShape<B, K>::NB];
            block_max<B, K>(v, m);
            quantize_values<FMT, B, K, MSE, DQ>(p, u, v, m, lane, kc, tab, nz, acc, pol);
        },
        MSE, pol);
    if constexpr (MSE) {
        cta_partials(acc[0], acc[0] - acc[1] - acc[2], acc[1], acc[2], p.partials);
        finish_partials(p.partials, p.done, p.n, p.terms);
    }
}

// max |y| of the rotated tensor (K = 16, 32) on the tensor cores.  The
// normalisation y = fp32(s / sqrt(K)) rounds monotonically in s, so the
// maximum is normalised once, after the maximum of the raw sums.
template <int K>
__global__ void __launch_bounds__(kThreads, 2) amax_tc_kernel(AmaxParams p)
{
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem_tc[];
    float mx = 0.0f;
    tc::rotate_tiles<K>(
        p.x, p.n, smem_tc, p.fault,
        [&](int64_t, f32x2 (&v)[EPT / 2]) { mx = fmaxf(mx, pairs_absmax<EPT>(v)); }, false, 0);
    f32x2 m2[1] = {pk(mx, mx)};
    normalize<2>(m2, p.c_hi, p.c_lo);
    float a, b;
    upk(m2[0], a, b);
    mx = group_max<32>(a);
    if ((threadIdx.x & 31) == 0 && mx > 0.0f) atomicMax(p.amax_bits, __float_as_uint(mx));
}

}  // namespace fp4q
