// fp4q_gemm.cu -- the block-scaled FP4 GEMM that consumes the quantizer's
// output: Y = G_A G_B (A_q . S_A) (B_q . S_B)^T on the 5th-generation tensor
// cores (tcgen05.mma kind::mxf4nvf4 block16 for NVFP4, kind::mxf4 block32 for
// MXFP4), fp32 accumulators in tensor memory.
//
// "Bridging the Gap", s3.4 and s4: the speed-ups of the pages come from FP4
// GEMMs that take the FP4 codes and block scales of both operands directly;
// "Diagnosing FP4 inference", Methodology: weights are quantized and then
// consumed by the compute.  The product computed is
//     Y[m][n] = G_A G_B sum_k q_A[m][k] s_A[m][k / b] q_B[n][k] s_B[n][k / b],
// q the E2M1 value of a code, s the decoded scale byte (UE4M3 or E8M0), both
// operands [rows][K] row-major with blocks of b along K (fp4q_quantize_mma's
// codes and MMA-layout scales).
//
// A persistent grid (one CTA per SM) walks the 128 x 128 tiles of Y; each
// tile walks K in stages of 256 elements (128 bytes of codes per row) through
// a ring of NSTAGE shared-memory stages:
//   warp 0, one thread: TMA loads of the A and B code tiles (128-byte swizzle,
//     straight into the layout the MMA reads) and bulk copies of the scale
//     atoms, completing on the stage's `full` mbarrier;
//   warp 1: allocates tensor memory; one thread copies each stage's scale
//     atoms into tensor memory (tcgen05.cp) and issues the MMAs into one of
//     two accumulator buffers (alternating tile by tile), releasing the stage
//     through its `empty` mbarrier (tcgen05.commit) and, after a tile's last
//     stage, the buffer through `afull`;
//   warps 2-5: the epilogue, each reading its 32 accumulator lanes
//     (tcgen05.ld), handing the buffer back (`aempty`), scaling by G_A G_B and
//     storing fp32 rows of Y -- while the MMAs of the next tile run into the
//     other buffer.
// Every wait is bounded; a wait that runs out records the library's fault word
// and the CTA stops its work and returns.
#include <cuda.h>

#include <mutex>

#include "fp4q_device.cuh"
#include "fp4q_launch.h"
#include "fp4q_tc.cuh"
#include "../../include/fp4q.h"

namespace fp4q {
namespace gemm {

constexpr int BM = 128, BN = 128;
constexpr int BK = 256;                     // elements of K per stage
constexpr int BKB = BK / 2;                 // bytes of codes per row per stage (one 128-byte swizzle row)
constexpr int NSTAGE = 4;
constexpr int A_BYTES = BM * BKB;           // 16 KiB
constexpr int B_BYTES = BN * BKB;           // 16 KiB
constexpr int SF_BYTES = 4 * 512;           // at most 4 scale atoms per operand per stage
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + 2 * SF_BYTES;   // 36 KiB
constexpr int SMEM_BYTES = 1024 + NSTAGE * STAGE_BYTES + 256;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr uint32_t TMEM_COLS = 512;         // two 128-column accumulators + the scale ring, NSTAGE x 32
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SF_COL = 2 * BN;
static_assert(SF_COL + NSTAGE * 32 <= TMEM_COLS, "tensor memory: accumulators and scale ring");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
constexpr uint32_t kMaxPolls = 1u << 24;

struct Params {
    CUtensorMap ta;                 // A codes [m][k / 2] bytes, box 128 x 128, 128-byte swizzle
    CUtensorMap tb;                 // B codes [n][k / 2]
    const uint8_t* sfa;             // A scales, MMA layout
    const uint8_t* sfb;
    const float* ga;                // per-tensor scales (nullptr: 1)
    const float* gb;
    float* y;                       // [m][n] fp32
    int64_t m, n, k;
    int64_t sf_kt;                  // 512-byte scale atoms per 128-row block
    int nvfp4;                      // 1: UE4M3 scales, block 16; 0: E8M0, block 32
    unsigned int* fault;
};

// K-major operand in the 128-byte swizzle layout (rows of 128 bytes, 8-row
// groups 1024 bytes apart): start >> 4, leading offset 1, stride 1024 >> 4,
// version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t a)
{
    return (uint64_t)((a >> 4) & 0x3fffu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// A 32-row x 16-byte scale atom in shared memory (no swizzle: 8-row core
// matrices 128 bytes apart) as the source of tcgen05.cp.
__device__ __forceinline__ uint64_t atom_desc(uint32_t a)
{
    return (uint64_t)((a >> 4) & 0x3fffu) | ((uint64_t)1u << 16) | ((uint64_t)(128u >> 4) << 32) |
           ((uint64_t)1u << 46);
}

// Block-scaled instruction descriptor: A and B E2M1 (bits 7-9, 10-12 = 1),
// K-major, N >> 3 in bits 17-22, scale type in bit 23 (0 UE4M3, 1 UE8M0),
// M >> 4 in bits 24-28, the scale byte of A in bits 29-30 and of B in 4-5.
__device__ __forceinline__ uint32_t bs_idesc(bool nvfp4, uint32_t sf_id)
{
    return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((nvfp4 ? 0u : 1u) << 23) |
           ((uint32_t)(BM >> 4) << 24) | (sf_id << 29) | (sf_id << 4);
}

__device__ __forceinline__ void mma_nvfp4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, bool acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
                 ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"((uint32_t)acc)
                 : "memory");
}

__device__ __forceinline__ void mma_mxfp4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, bool acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
                 ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"((uint32_t)acc)
                 : "memory");
}

// 32 rows x 128 bits of shared memory into 4 tensor-memory columns of the 32
// lanes, repeated in all four 32-lane quarters.
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Bounded wait on an mbarrier phase; false (and the fault word set) when it runs out.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, unsigned int* fault)
{
    for (uint32_t polls = 0; polls < kMaxPolls; ++polls)
        if (tc::mbar_try_wait(bar, parity)) return true;
    atomicExch(fault, 1u);
    return false;
}

__global__ void __launch_bounds__(THREADS, 1) fp4_gemm_kernel(const __grid_constant__ Params p)
{
    extern __shared__ __align__(1024) uint8_t smem_g[];
    const uint32_t raw = (uint32_t)__cvta_generic_to_shared(smem_g);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t bars = base + NSTAGE * STAGE_BYTES;
    const uint32_t full0 = bars, empty0 = full0 + 8u * NSTAGE;
    const uint32_t afull0 = empty0 + 8u * NSTAGE, aempty0 = afull0 + 16u;   // 2 accumulator buffers
    const uint32_t slot = aempty0 + 16u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int64_t tiles_n = (p.n + BN - 1) / BN;
    const int64_t n_tiles = ((p.m + BM - 1) / BM) * tiles_n;
    const int64_t kt_n = (p.k + BK - 1) / BK;              // stages of K per tile (the last may be partial)
    const int apk = p.nvfp4 ? 4 : 2;                         // scale atoms per full stage per operand

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            tc::mbar_init(full0 + 8u * i, 1u);
            tc::mbar_init(empty0 + 8u * i, 1u);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(afull0 + 8u * i, 1u);
            tc::mbar_init(aempty0 + 8u * i, (uint32_t)EPI_WARPS);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tc::tmem_alloc(slot, TMEM_COLS);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(slot) : "memory");

    if (warp == 0 && lane == 0) {
        // ---- producer: the (tile, k-stage) sequence of this CTA through the ring
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.ta)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tb)) : "memory");
        int64_t g = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            const int64_t m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
            for (int64_t kt = 0; kt < kt_n; ++kt, ++g) {
                const int s = (int)(g % NSTAGE);
                if (g >= NSTAGE && !wait_phase(empty0 + 8u * s, (uint32_t)(((g / NSTAGE) - 1) & 1), p.fault)) {
                    ok = false;
                    break;
                }
                const int steps = (int)((p.k - kt * BK) >= BK ? 4 : (p.k - kt * BK) / 64);
                const int64_t atom0 = kt * apk;
                int natoms = p.nvfp4 ? steps : (steps + 1) / 2;
                if (atom0 + natoms > p.sf_kt) natoms = (int)(p.sf_kt - atom0);
                const uint32_t st = base + (uint32_t)(s * STAGE_BYTES);
                const uint32_t fb = full0 + 8u * s;
                mbar_expect_tx(fb, (uint32_t)(A_BYTES + B_BYTES + 2 * natoms * 512));
                tma_load_2d(st, &p.ta, (int)(kt * BKB), (int)m0, fb);
                tma_load_2d(st + A_BYTES, &p.tb, (int)(kt * BKB), (int)n0, fb);
                const uint8_t* sa = p.sfa + (((m0 >> 7) * p.sf_kt + atom0) << 9);
                const uint8_t* sb = p.sfb + (((n0 >> 7) * p.sf_kt + atom0) << 9);
                bulk_load(st + A_BYTES + B_BYTES, sa, (uint32_t)natoms * 512u, fb);
                bulk_load(st + A_BYTES + B_BYTES + SF_BYTES, sb, (uint32_t)natoms * 512u, fb);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---- scale copies and MMAs, one accumulator buffer per tile, alternating
        int64_t g = 0, j = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++j) {
            const int ab = (int)(j & 1);
            if (j >= 2 && !wait_phase(aempty0 + 8u * ab, (uint32_t)(((j >> 1) - 1) & 1), p.fault)) break;
            const uint32_t acc_col = tmem + ACC_COL + (uint32_t)(ab * BN);
            for (int64_t kt = 0; kt < kt_n; ++kt, ++g) {
                const int s = (int)(g % NSTAGE);
                if (!wait_phase(full0 + 8u * s, (uint32_t)((g / NSTAGE) & 1), p.fault)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const int steps = (int)((p.k - kt * BK) >= BK ? 4 : (p.k - kt * BK) / 64);
                const int64_t atom0 = kt * apk;
                int natoms = p.nvfp4 ? steps : (steps + 1) / 2;
                if (atom0 + natoms > p.sf_kt) natoms = (int)(p.sf_kt - atom0);
                const uint32_t st = base + (uint32_t)(s * STAGE_BYTES);
                const uint32_t sf_a = tmem + SF_COL + 32u * (uint32_t)s;     // 4 columns per atom
                const uint32_t sf_b = sf_a + 16u;
                for (int a = 0; a < natoms; ++a) {
                    tmem_cp_atom(sf_a + 4u * a, atom_desc(st + A_BYTES + B_BYTES + 512u * a));
                    tmem_cp_atom(sf_b + 4u * a, atom_desc(st + A_BYTES + B_BYTES + SF_BYTES + 512u * a));
                }
                for (int kk = 0; kk < steps; ++kk) {
                    const uint64_t da = sw128_desc(st + 32u * kk);
                    const uint64_t db = sw128_desc(st + A_BYTES + 32u * kk);
                    const bool acc = kt > 0 || kk > 0;
                    if (p.nvfp4) {
                        mma_nvfp4(acc_col, da, db, bs_idesc(true, 0), sf_a + 4u * kk, sf_b + 4u * kk, acc);
                    } else {
                        const uint32_t id = 2u * (uint32_t)(kk & 1);
                        const uint32_t col = 4u * (uint32_t)(kk >> 1);
                        mma_mxfp4(acc_col, da, db, bs_idesc(false, id), (sf_a + col) | (id << 30),
                                  (sf_b + col) | (id << 30), acc);
                    }
                }
                tc::mma_commit(empty0 + 8u * s);        // the stage (smem and its scale columns) is free again
            }
            if (ok) tc::mma_commit(afull0 + 8u * ab);   // the tile's accumulator is complete
        }
    } else if (warp >= 2) {
        // ---- epilogue: warp w reads accumulator lanes 32 (w % 4) .. + 31
        const int q = warp & 3;
        const float g = (p.ga ? *p.ga : 1.0f) * (p.gb ? *p.gb : 1.0f);
        int64_t j = 0;
        for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++j) {
            const int ab = (int)(j & 1);
            const bool done = wait_phase(afull0 + 8u * ab, (uint32_t)((j >> 1) & 1), p.fault);
            if (!__all_sync(0xffffffffu, done)) break;
            tc::tc_fence_after();
            const int64_t m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
            const int64_t r = m0 + 32 * q + lane;
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + ACC_COL + (uint32_t)(ab * BN) + 32u * (uint32_t)c,
                              v);
                if (c == BN / 32 - 1) {
                    // every column of this warp's lanes is in registers: the buffer may be refilled
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(aempty0 + 8u * ab);
                }
                const int64_t c0 = n0 + 32 * c;
                if (r < p.m && c0 < p.n) {
                    float* dst = p.y + r * p.n + c0;
                    if (c0 + 32 <= p.n && (p.n & 3) == 0) {
#pragma unroll
                        for (int jj = 0; jj < 32; jj += 4)
                            stg128(dst + jj, __float_as_uint(__fmul_rn(__uint_as_float(v[jj]), g)),
                                   __float_as_uint(__fmul_rn(__uint_as_float(v[jj + 1]), g)),
                                   __float_as_uint(__fmul_rn(__uint_as_float(v[jj + 2]), g)),
                                   __float_as_uint(__fmul_rn(__uint_as_float(v[jj + 3]), g)));
                    } else {
                        for (int jj = 0; jj < 32 && c0 + jj < p.n; ++jj)
                            dst[jj] = __fmul_rn(__uint_as_float(v[jj]), g);
                    }
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// The driver's cuTensorMapEncodeTiled, fetched once at run time (the library
// links the runtime only).
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

// The code tiles of an operand: [rows][k / 2] bytes, boxes of 128 rows x 128
// bytes (one 128-byte swizzle row per K stage), 128-byte swizzle.
bool make_code_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t k)
{
    EncodeTiledFn enc = encode_fn();
    const uint64_t inner = (uint64_t)(k / 2);
    if (!enc || rows <= 0 || inner == 0) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)inner};
    const cuuint32_t box[2] = {(cuuint32_t)BKB, (cuuint32_t)BM};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gemm
}  // namespace fp4q

extern "C" int fp4q_gemm(const uint8_t* codes_a, const uint8_t* scales_a, const float* gscale_a, int64_t m,
                         const uint8_t* codes_b, const uint8_t* scales_b, const float* gscale_b, int64_t n,
                         int64_t k, int fmt, float* y, void* stream)
{
    using namespace fp4q;
    if (m < 0 || n < 0 || k < 0 || k % 64 != 0) return FP4Q_ERR_SHAPE;
    if (fmt != FP4Q_SCALE_E8M0 && fmt != FP4Q_SCALE_UE4M3) return FP4Q_ERR_UNSUPPORTED;
    if (fmt == FP4Q_SCALE_E8M0 && (gscale_a || gscale_b)) return FP4Q_ERR_UNSUPPORTED;
    if (m == 0 || n == 0) return FP4Q_OK;
    if (!y) return FP4Q_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(y) & 15u) != 0) return FP4Q_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (k == 0) return cudaMemsetAsync(y, 0, (size_t)(m * n) * sizeof(float), s) == cudaSuccess ? FP4Q_OK
                                                                                            : FP4Q_ERR_CUDA;
    if (!codes_a || !codes_b || !scales_a || !scales_b) return FP4Q_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(codes_a) & 15u) || (reinterpret_cast<uintptr_t>(codes_b) & 15u) ||
        (reinterpret_cast<uintptr_t>(scales_a) & 15u) || (reinterpret_cast<uintptr_t>(scales_b) & 15u))
        return FP4Q_ERR_ALIGN;
    if ((gscale_a && (reinterpret_cast<uintptr_t>(gscale_a) & 3u)) ||
        (gscale_b && (reinterpret_cast<uintptr_t>(gscale_b) & 3u)))
        return FP4Q_ERR_ALIGN;
    gemm::Params p;
    memset(&p, 0, sizeof(p));
    if (!gemm::make_code_map(&p.ta, codes_a, m, k) || !gemm::make_code_map(&p.tb, codes_b, n, k))
        return FP4Q_ERR_CUDA;
    const int block = fmt == FP4Q_SCALE_UE4M3 ? 16 : 32;
    p.sfa = scales_a;
    p.sfb = scales_b;
    p.ga = gscale_a;
    p.gb = gscale_b;
    p.y = y;
    p.m = m;
    p.n = n;
    p.k = k;
    p.sf_kt = (k / block + 3) / 4;
    p.nvfp4 = fmt == FP4Q_SCALE_UE4M3;
    p.fault = device_fault_word();
    if (!p.fault) return FP4Q_ERR_CUDA;
    const int64_t tiles = ((m + gemm::BM - 1) / gemm::BM) * ((n + gemm::BN - 1) / gemm::BN);
    const int grid = grid_for((const void*)gemm::fp4_gemm_kernel, gemm::SMEM_BYTES, tiles, gemm::THREADS);
    gemm::fp4_gemm_kernel<<<grid, gemm::THREADS, gemm::SMEM_BYTES, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA;
}
