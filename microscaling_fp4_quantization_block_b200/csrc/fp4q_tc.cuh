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
// lands in TMEM lane m, so after one tcgen05.ld each thread of a consumer warp
// holds the 32 rotated values of "its" row: the same 32-element unit the
// quantizer works on, with no shuffles.
//
// Warp-specialised pipeline (a CTA of 4 consumer warps, a producer warp and an
// MMA warp; the two single-thread roles sit in different warps so that a
// blocking mbarrier probe in one never stalls the other):
//   producer warp, one thread: TMA loads of 4096-element tiles (a 2-D tensor
//     map of 64-byte rows with the 64-byte swizzle, which is the K-major layout
//     the MMA reads) into a ring of NSTAGE shared-memory stages, completing on
//     the stage's `full` mbarrier;
//   MMA warp, one thread: per tile, the two K = 16 MMAs into one of NBUF TMEM
//     accumulator buffers, then tcgen05.commit on the stage's `empty` barrier
//     (the stage may be refilled) and the buffer's `tfull` barrier;
//   consumer warps: per tile, wait for `tfull`, tcgen05.ld their 32 lanes,
//     arrive on the buffer's `tempty` barrier (4 arrivals free it), quantize.
// No barrier couples the consumer warps to one another, so each runs ahead as
// far as the pipeline allows.  Every wait is bounded; one that runs out sets
// the library's fault word (fp4q_device_fault) and that role stops its work.
#pragma once

#include <cuda.h>

#include "fp4q_kernels.cuh"

namespace fp4q {
namespace tc {

constexpr int KR = 32;                          // elements per MMA row
constexpr int ROWS = 128;                       // rows per tile (M of the MMA), one per consumer thread
constexpr int TILE_ELEMS = ROWS * KR;           // 4096
constexpr int STAGE_BYTES = ROWS * KR * 2;      // 8 KiB of bf16
constexpr int NSTAGE = 6;                       // shared-memory ring stages
constexpr int NBUF = 4;                         // TMEM accumulator buffers of 32 columns
constexpr int CONSUMER_WARPS = 4;
constexpr int PRODUCER_WARP = CONSUMER_WARPS;   // TMA loads
constexpr int MMA_WARP = CONSUMER_WARPS + 1;    // TMEM allocation and the MMAs
constexpr int THREADS = 32 * (CONSUMER_WARPS + 2);
constexpr int TMEM_COLS = NBUF * KR;            // 128 (a power of two >= 32)
constexpr int B_BYTES = KR * KR * 2;            // the rotation matrix, 2 KiB
// dynamic shared memory: 1 KiB of slack to align the swizzled buffers to 1 KiB,
// the rotation matrix, the ring, then the mbarriers and the TMEM address slot
constexpr int SMEM_BYTES = 1024 + B_BYTES + NSTAGE * STAGE_BYTES + 8 * (2 * NSTAGE + 2 * NBUF) + 16;

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
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, int x, int y, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
                 : "memory");
}

// Bounded wait on an mbarrier phase; false (and the fault word set) when it runs out.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, unsigned int* fault)
{
    for (uint32_t polls = 0; polls < kMaxPolls; ++polls)
        if (mbar_try_wait(bar, parity)) return true;
    atomicExch(fault, 1u);
    return false;
}

// Every 4096-element tile of x (bf16, n elements, n a multiple of 32, read
// through the tensor map xmap: rows of 32 elements, boxes of 128 rows) is
// rotated by the tensor cores; body(u, v) is then called by every consumer
// thread for unit u (32 consecutive elements, u = tile * 128 + row) with the
// rotated, not yet normalised, values v.  Rows at or past n read as zeros.
// CTAs walk tiles in a grid-stride loop.  Called by all THREADS threads.
template <int K, typename Body>
__device__ __forceinline__ void rotate_tiles(const void* xmap, int64_t n, uint8_t* smem_raw, unsigned int* fault,
                                             Body&& body)
{
    const uint32_t raw = (uint32_t)__cvta_generic_to_shared(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;               // swizzle atoms need 1 KiB alignment
    const uint32_t b_smem = base;
    const uint32_t ring = base + B_BYTES;
    const uint32_t bars = ring + NSTAGE * STAGE_BYTES;
    const uint32_t full0 = bars, empty0 = full0 + 8u * NSTAGE;
    const uint32_t tfull0 = empty0 + 8u * NSTAGE, tempty0 = tfull0 + 8u * NBUF;
    const uint32_t slot = tempty0 + 8u * NBUF;                  // TMEM base address
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    fill_rotation_matrix<K>(b_smem);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(full0 + 8u * i, 1u);
            mbar_init(empty0 + 8u * i, 1u);
        }
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(tfull0 + 8u * i, 1u);
            mbar_init(tempty0 + 8u * i, (uint32_t)CONSUMER_WARPS);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == MMA_WARP) tmem_alloc(slot, TMEM_COLS);
    fence_proxy_async_smem();                                    // the rotation matrix, for the MMA
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t tmem_base;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem_base) : "r"(slot) : "memory");

    const int64_t n_tiles = (n + TILE_ELEMS - 1) / TILE_ELEMS;
    const int64_t first = blockIdx.x, stride = gridDim.x;

    if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            // ---- TMA producer
            int64_t i = 0;
            for (int64_t t = first; t < n_tiles; t += stride, ++i) {
                const int s = (int)(i % NSTAGE);
                if (i >= NSTAGE && !wait_bounded(empty0 + 8u * s, (uint32_t)(((i / NSTAGE) - 1) & 1), fault)) break;
                mbar_expect_tx(full0 + 8u * s, (uint32_t)STAGE_BYTES);
                tma_load_2d(ring + (uint32_t)(s * STAGE_BYTES), xmap, 0, (int)(t * ROWS), full0 + 8u * s);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            // ---- MMA issuer
            int64_t i = 0;
            for (int64_t t = first; t < n_tiles; t += stride, ++i) {
                const int s = (int)(i % NSTAGE), b = (int)(i % NBUF);
                if (!wait_bounded(full0 + 8u * s, (uint32_t)((i / NSTAGE) & 1), fault)) break;
                if (i >= NBUF && !wait_bounded(tempty0 + 8u * b, (uint32_t)(((i / NBUF) - 1) & 1), fault)) break;
                tc_fence_after();
                const uint32_t a = ring + (uint32_t)(s * STAGE_BYTES);
                const uint32_t d = tmem_base + (uint32_t)(b * KR);
                mma_bf16(d, sw64_desc(a), sw64_desc(b_smem), kIdescBf16F32, false);
                mma_bf16(d, sw64_desc(a + 32u), sw64_desc(b_smem + 32u), kIdescBf16F32, true);
                mma_commit(empty0 + 8u * s);                    // the stage may be refilled
                mma_commit(tfull0 + 8u * b);                    // the buffer may be read
            }
        }
        __syncwarp();
    } else {
        // ---- consumers: warp w reads TMEM lanes 32 w .. 32 w + 31 (rows of the tile)
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
        int64_t i = 0;
        for (int64_t t = first; t < n_tiles; t += stride, ++i) {
            const int b = (int)(i % NBUF);
            const bool done = mbar_try_wait(tfull0 + 8u * b, (uint32_t)((i / NBUF) & 1)) ||
                              wait_bounded(tfull0 + 8u * b, (uint32_t)((i / NBUF) & 1), fault);
            if (!__all_sync(0xffffffffu, done)) break;         // warp-uniform: tcgen05.ld needs the warp
            tc_fence_after();
            uint32_t r[32];
            tmem_ld32(tmem_base + lane_off + (uint32_t)(b * KR), r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty0 + 8u * b);      // this warp is done with the buffer
            f32x2 v[EPT / 2];
#pragma unroll
            for (int k = 0; k < EPT / 2; ++k) v[k] = pk(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
            body(t * ROWS + 32 * warp + lane, v);
        }
    }
    // every MMA issued has completed (each was waited on by the consumers, or a
    // role gave up), so TMEM can be released
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace tc

// ---------------------------------------------------------------- kernels on the tensor-core rotation
// Parameters: the quantizer's (or the maximum's) plus the tensor map of x.
struct TcQuantParams {
    CUtensorMap xmap;
    QuantParams p;
};

struct TcAmaxParams {
    CUtensorMap xmap;
    AmaxParams p;
};

// Quantize (+ fused MSE / dequantized output) with the rotation (K = 16, 32)
// on the tensor cores; outputs identical in layout to quantize_kernel's.
template <int FMT, int B, int K, bool MSE, bool DQ>
__global__ void __launch_bounds__(tc::THREADS, 3) quantize_tc_kernel(const __grid_constant__ TcQuantParams tp)
{
    static_assert(K == 16 || K == 32, "tensor-core rotation of 16 or 32");
    const QuantParams& p = tp.p;
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
    tc::rotate_tiles<K>(&tp.xmap, p.n, smem_tc, p.fault, [&](int64_t u, f32x2 (&v)[EPT / 2]) {
        normalize<EPT>(v, p.c_hi, p.c_lo);
        float m[UnitShape<B, K>::NB];
        block_max<B, K>(v, m);
        quantize_values<FMT, B, K, MSE, DQ>(p, u, v, m, lane, kc, tab, nz, acc, pol);
    });
    if constexpr (MSE) {
        cta_partials<tc::THREADS>(acc[0], acc[0] - acc[1] - acc[2], acc[1], acc[2], p.partials);
        finish_partials<tc::THREADS>(p.partials, p.done, p.n, p.terms);
    }
}

// max |y| of the rotated tensor (K = 16, 32) on the tensor cores.  The
// normalisation y = fp32(s / sqrt(K)) rounds monotonically in s, so the
// maximum is normalised once, after the maximum of the raw sums.
template <int K>
__global__ void __launch_bounds__(tc::THREADS, 3) amax_tc_kernel(const __grid_constant__ TcAmaxParams tp)
{
    const AmaxParams& p = tp.p;
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(128) uint8_t smem_tc[];
    float mx = 0.0f;
    tc::rotate_tiles<K>(&tp.xmap, p.n, smem_tc, p.fault,
                        [&](int64_t, f32x2 (&v)[EPT / 2]) { mx = fmaxf(mx, pairs_absmax<EPT>(v)); });
    f32x2 m2[1] = {pk(mx, mx)};
    normalize<2>(m2, p.c_hi, p.c_lo);
    float a, b;
    upk(m2[0], a, b);
    mx = group_max<32>(a);
    if ((threadIdx.x & 31) == 0 && mx > 0.0f) atomicMax(p.amax_bits, __float_as_uint(mx));
}

}  // namespace fp4q
