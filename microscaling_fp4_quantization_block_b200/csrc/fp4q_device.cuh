// fp4q_device.cuh -- device building blocks of the FP4 block quantizer (sm_100a).
//
// Number formats ("Diagnosing FP4 inference", Methodology; "Bridging the Gap",
// s1; "Finer is better?", Theoretical framework and Contributions):
//   E2M1 element: sign, 2 exponent bits (bias 1), 1 mantissa bit: magnitudes
//     {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
//   E8M0 scale: 2^(byte - 127).
//   UE4M3 scale: unsigned E4M3, bias 7, 0x7F NaN, max 448, min 2^-9.
//   UE5M3 scale: unsigned E5M3, bias 15, 0xFF NaN, max 114688, min 2^-17.
// The library is built with -fmad=false: every a*b+c below is two roundings
// unless it is written as an explicit fused multiply-add.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace fp4q {

enum ScaleFmt : int { kE8M0 = 0, kUE4M3 = 1, kUE5M3 = 2 };

// ---------------------------------------------------------------- bit casts
__device__ __forceinline__ float as_f32(uint32_t b) { return __uint_as_float(b); }
__device__ __forceinline__ uint32_t as_u32(float f) { return __float_as_uint(f); }

// Two bf16 values packed in one 32-bit word (element 2i in the low half):
// widening to fp32 is exact and is just a shift / mask.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return as_f32(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return as_f32(w & 0xffff0000u); }

// The high half widened by a mixed-precision add of -0 (bf16 + fp32 -> fp32,
// exact): it issues on the floating-point pipe instead of the integer/logic
// pipe that the mask above uses, which the rest of the quantizer keeps busy.
__device__ __forceinline__ float bf16_hi_fp(uint32_t w)
{
    float r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, h, %2;\n\t}"
        : "=f"(r)
        : "r"(w), "f"(-0.0f));
    return r;
}

// Per half, max(|a|, |b|) of two bf16x2 words; the result's sign bits are
// meaningless (xor of the inputs' signs) and are dropped by bf16x2_absmax_f32.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Larger magnitude of the two halves of a bf16x2 word, as fp32 (exact).
__device__ __forceinline__ float bf16x2_absmax_f32(uint32_t m)
{
    return fmaxf(as_f32((m << 16) & 0x7fffffffu), as_f32(m & 0x7fff0000u));
}

// ---------------------------------------------------------------- vector memory
struct alignas(32) U32x8 { uint32_t v[8]; };

// 256-bit global load, read-only path, no L1 allocation (streamed once).
__device__ __forceinline__ U32x8 ldg256_stream(const void* p)
{
    U32x8 r;
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r.v[0]), "=r"(r.v[1]), "=r"(r.v[2]), "=r"(r.v[3]),
                   "=r"(r.v[4]), "=r"(r.v[5]), "=r"(r.v[6]), "=r"(r.v[7])
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void stg128(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ void stg256(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                       uint32_t f, uint32_t g, uint32_t h)
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d),
                 "r"(e), "r"(f), "r"(g), "r"(h)
                 : "memory");
}

// ---------------------------------------------------------------- L2 eviction priority
// A cache policy under which the lines an access allocates in L2 are the
// first to go.  Outputs, and the last read of an input, use it so that they
// do not push out input lines that a later pass of the same step will read.
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void stg128(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void stg256(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                       uint32_t f, uint32_t g, uint32_t h, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8}, %9;" ::"l"(p), "r"(a), "r"(b),
                 "r"(c), "r"(d), "r"(e), "r"(f), "r"(g), "r"(h), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void stg64(void* p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

// ---------------------------------------------------------------- programmatic dependent launch
// Wait until the grids this one depends on have completed and their memory is
// visible (a no-op for a plain launch), then let the next grid in the stream
// be scheduled as this one's CTAs retire.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- async copies into shared memory
// 16-byte global -> shared copy (L2 only, no L1); src_bytes 0 writes zeros and
// reads nothing.  Completion is tracked per thread with commit / wait groups.
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr), "l"(gptr), "r"(src_bytes)
                 : "memory");
}
// The same copy, its L2 lines allocated under the cache policy pol.
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr, uint32_t src_bytes, uint64_t pol)
{
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(smem_addr), "l"(gptr),
                 "r"(src_bytes), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t smem_addr)
{
    uint4 r;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(smem_addr));
    return r;
}

// ---------------------------------------------------------------- E2M1
// Four pairs -> one 32-bit word of nibbles: byte k = code(v[2k]) | code(v[2k+1]) << 4.
// cvt.rn.satfinite.e2m1x2.f32 rounds to nearest even onto the E2M1 grid,
// saturates at +-6 and keeps the sign; its first source lands in the high nibble.
__device__ __forceinline__ uint32_t e2m1_pack8(float v0, float v1, float v2, float v3, float v4,
                                               float v5, float v6, float v7)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return r;
}

// Codes of 8 values -> code word, plus each code byte decoded back to an
// f16x2 pair (h[j] = grid values of elements 2j, 2j+1) for the MSE.
__device__ __forceinline__ uint32_t e2m1_pack8_dec(float v0, float v1, float v2, float v3, float v4, float v5,
                                                   float v6, float v7, uint32_t (&h)[4])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %8, %7;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %12, %11;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %4, b3;\n\t}"
        : "=r"(r), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return r;
}

// Two nibbles (one code byte, low nibble first) -> two exact fp32 values.
__device__ __forceinline__ void e2m1_unpack2(uint32_t byte, float& lo, float& hi)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.u8.u32 b, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
        : "=r"(h2)
        : "r"(byte));
    // f16x2: low half = low nibble
    __half2 hh = *reinterpret_cast<__half2*>(&h2);
    lo = __low2float(hh);
    hi = __high2float(hh);
}

// Magnitude of the E2M1 grid value that q rounds to (E2M1 code, then its
// value, through the two hardware conversions).
__device__ __forceinline__ float e2m1_grid_value(float q)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %1, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
        : "=r"(h2)
        : "f"(q));
    return fabsf(__half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu))));
}

// ---------------------------------------------------------------- E8M0
// Scale byte for a block with absolute maximum m (m >= 0):
// 2^(floor(log2 m) - 2), floor(log2 m) read from the fp32 exponent field; a
// subnormal or zero m, and any m below 2^-125, clamps to byte 0 (2^-127).
__device__ __forceinline__ uint32_t e8m0_from_amax(float m)
{
    uint32_t e = as_u32(m) >> 23;                  // biased exponent (m >= 0)
    if (e == 0xffu) return 0xffu;                  // non-finite input: NaN scale
    return e >= 2u ? e - 2u : 0u;
}

// 2^(byte-127) as fp32 (byte 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_decode(uint32_t c)
{
    if (c == 0u) return as_f32(0x00400000u);
    if (c == 0xffu) return as_f32(0x7fc00000u);
    return as_f32(c << 23);
}

// 1 / 2^(byte-127), exact for bytes 0..253 (the only ones finite inputs produce).
__device__ __forceinline__ float e8m0_inverse(uint32_t c)
{
    if (c >= 254u) return as_f32(0x7fc00000u);
    return as_f32((254u - c) << 23);
}

// ---------------------------------------------------------------- UE4M3
// Nearest UE4M3 code to s >= 0: the hardware E4M3 conversion (round to nearest
// even, saturate to 448, NaN -> 0x7F); s >= 0 keeps the sign bit clear.
__device__ __forceinline__ uint32_t ue4m3_encode(float s)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
    return (uint32_t)(r & 0xffu);
}

// Two UE4M3 codes at once: low byte = code(a), high byte = code(b).
__device__ __forceinline__ uint32_t ue4m3_encode2(float a, float b)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return (uint32_t)r;
}

__device__ __forceinline__ float ue4m3_decode(uint32_t c)
{
    uint32_t e = c >> 3, m = c & 7u;
    if (c >= 0x7fu) return as_f32(0x7fc00000u);
    if (e == 0u) return __fmul_rn((float)m, 0.001953125f);          // m * 2^-9, exact
    return as_f32(((e + 120u) << 23) | (m << 20));
}

// The same decode through the hardware E4M3 -> f16 conversion (exact: every
// UE4M3 value is an f16 value), for codes 0..0x7E.
__device__ __forceinline__ float ue4m3_decode_hw(uint32_t c)
{
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(c));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// Two UE4M3 codes (low byte first) -> two exact fp32 values, one conversion.
__device__ __forceinline__ void ue4m3_decode2_hw(uint32_t c2, float& lo, float& hi)
{
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(c2));
    lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
    hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// ---------------------------------------------------------------- UE5M3
// Nearest UE5M3 code to s >= 0 by integer rounding of the fp32 pattern: keep 3
// mantissa bits with round-to-nearest-even (a carry moves into the exponent);
// below the smallest normal (2^-14) the code is the nearest multiple of 2^-17;
// above the largest finite value (0xFE) saturate.
__device__ __forceinline__ uint32_t ue5m3_encode(float s)
{
    uint32_t b = as_u32(s);
    if (b >= 0x7f800000u) return (b > 0x7f800000u) ? 0xffu : 0xfeu;   // NaN / +inf
    if (b == 0u) return 0u;
    uint32_t e = b >> 23;
    if (e >= 113u) {                                                   // >= 2^-14: normal target
        uint32_t mant = b & 0x7fffffu;
        uint32_t q = ((e - 112u) << 3) | (mant >> 20);
        uint32_t rnd = (mant >> 19) & 1u, sticky = mant & 0x7ffffu;
        if (rnd && (sticky || (q & 1u))) q += 1u;
        return q > 0xfeu ? 0xfeu : q;
    }
    // subnormal target: code = RNE(s * 2^17), at most 8 (= the smallest normal)
    float t = __fmul_rn(s, 131072.0f);
    return (uint32_t)__float2int_rn(t);
}

__device__ __forceinline__ float ue5m3_decode(uint32_t c)
{
    uint32_t e = c >> 3, m = c & 7u;
    if (c >= 0xffu) return as_f32(0x7fc00000u);
    if (e == 0u) return __fmul_rn((float)m, 7.62939453125e-06f);     // m * 2^-17, exact
    return as_f32(((e + 112u) << 23) | (m << 20));
}

// ---------------------------------------------------------------- packed fp32 pairs
// sm_100 executes two fp32 operations per instruction on a 64-bit register
// pair (add/sub/mul/fma .rn.f32x2); each lane of the pair rounds exactly like
// the scalar instruction.  Unlike the scalar .rn forms, a packed product that
// feeds a packed add or subtract may be fused into one multiply-add by the
// assembler, so a product whose own rounding matters (a dequantized value
// that is then subtracted or rotated) is formed with mul2_rounded instead.
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pk(float a, float b)
{
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(f32x2 v, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

// 16 bytes of shared memory as two fp32 pairs, and back.
__device__ __forceinline__ void sts_pairs(uint32_t smem_addr, f32x2 a, f32x2 b)
{
    asm volatile("st.shared.v2.b64 [%0], {%1, %2};" ::"r"(smem_addr), "l"(a), "l"(b) : "memory");
}
__device__ __forceinline__ void lds_pairs(uint32_t smem_addr, f32x2& a, f32x2& b)
{
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(smem_addr) : "memory");
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// Two products, each rounded to fp32 on its own (scalar .rn multiplies are never
// contracted into a following add).
__device__ __forceinline__ f32x2 mul2_rounded(f32x2 a, f32x2 b)
{
    float a0, a1, b0, b1;
    upk(a, a0, a1);
    upk(b, b0, b1);
    return pk(__fmul_rn(a0, b0), __fmul_rn(a1, b1));
}

// a * b + c with one rounding toward minus infinity, on both lanes.
__device__ __forceinline__ f32x2 fma2_rm(f32x2 a, f32x2 b, f32x2 c)
{
    f32x2 r;
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b)
{
    f32x2 r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c)
{
    f32x2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// max(|a|, |b|, |c|) in one three-input instruction (sm_100).
__device__ __forceinline__ float amax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// ---------------------------------------------------------------- correctly rounded quotients
// A quotient a / b that decides a code (element y / S, scale m / fp32(6G)) is
// computed exactly, without a divide, from the correctly rounded reciprocal
// R = fp32(1/b) (one per scale, not per element) by the remainder correction
// of Markstein's division theorem:
//   q0 = fp32(a R),   r = a - q0 b (exact; one fused multiply-add),
//   q  = fp32(q0 + r R)  =  fp32(a / b).
// The remainder is rounded toward minus infinity only so that an exact zero
// remainder is -0: then a = -0 gives q = -0 and keeps its sign, as a true
// division does; a non-zero remainder is exact and unaffected.  The identity is
// checked on the GPU exhaustively for every bf16 significand a against every
// fp32 significand b, both signs (the values the unrotated path divides), and
// on random fp32 pairs; it needs b, 1/b and the quotient normal, so callers
// keep b within [2^-100, 2^100] and |a / b| below 2^60 and divide otherwise.
__device__ __forceinline__ f32x2 div2_cr(f32x2 a, f32x2 R, f32x2 neg_b)
{
    const f32x2 q0 = mul2(a, R);
    const f32x2 r = fma2_rm(q0, neg_b, a);
    return fma2(r, R, q0);
}

constexpr float kDivLo = 0x1p-100f;     // range of divisors the remainder correction serves
constexpr float kDivHi = 0x1p100f;
constexpr float kQuotMax = 0x1p60f;

// Per-tensor constants of the UE scale rule: G, the divisor fp32(6G) of the
// block maxima and its correctly rounded reciprocal.
struct ScaleConsts {
    float G;
    float denom;             // fp32(6 G)
    float rdenom;            // fp32(1 / denom), when denom_ok
    bool denom_ok;           // denom within [2^-100, 2^100]
};

__device__ __forceinline__ ScaleConsts scale_consts(float G)
{
    ScaleConsts c;
    c.G = G;
    c.denom = __fmul_rn(6.0f, G);
    c.denom_ok = c.denom >= kDivLo && c.denom <= kDivHi;
    c.rdenom = c.denom_ok ? __frcp_rn(c.denom) : 0.0f;
    return c;
}

// ---------------------------------------------------------------- Hadamard
// Values are held as N/2 fp32 pairs p[k] = (v[2k], v[2k+1]).  In-register
// Sylvester Hadamard transform of every run of CH consecutive values (natural
// order: y_i = sum_j (-1)^popcount(i & j) x_j): the distance-1 stage mixes the
// two halves of each pair, the others combine whole pairs.  FIRST = false
// skips the distance-1 stage (done already by unpack_fwht2); the pair stages
// run at distances H0, 2 H0, ... below CH (H0 > 2: the stages of the lower
// index bits are done already).
template <int N, int CH, bool FIRST = true, int H0 = 2>
__device__ __forceinline__ void fwht_inreg(f32x2 (&p)[N / 2])
{
    if constexpr (FIRST && CH >= 2) {
#pragma unroll
        for (int k = 0; k < N / 2; ++k) {
            float a, b;
            upk(p[k], a, b);
            p[k] = pk(__fadd_rn(a, b), __fsub_rn(a, b));
        }
    }
#pragma unroll
    for (int h = H0; h < CH; h <<= 1) {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            if ((i & h) == 0) {
                const f32x2 a = p[i / 2], b = p[(i + h) / 2];
                p[i / 2] = add2(a, b);
                p[(i + h) / 2] = sub2(a, b);
            }
        }
    }
}

// bf16 words -> fp32 pairs with the distance-1 butterfly stage folded in:
// p[k] = (x0 + x1, x1 - x0) for w[k] = (x0, x1), each a single rounding of the
// exact sum or difference (mixed-precision add / subtract of the bf16 high
// half and the widened low half), so three instructions per pair instead of
// the widening (two) plus the stage (two).  The second value of every pair is
// the NEGATED distance-1 difference.  Every later stage, in registers or
// across lanes, combines like positions linearly, so the odd positions stay
// negated to the end of the transform, where the normalisation multiplies
// them by -c (RN(-a) = -RN(a): the values are exactly those of the plain
// transform).
template <int N>
__device__ __forceinline__ void unpack_fwht2(const uint32_t (&w)[N / 2], f32x2 (&p)[N / 2])
{
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
        const float lo = bf16_lo(w[k]);
        float s, d;
        asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tadd.rn.f32.bf16 %0, h, %3;\n\t"
            "sub.rn.f32.bf16 %1, h, %3;\n\t}"
            : "=f"(s), "=f"(d)
            : "r"(w[k]), "f"(lo));
        p[k] = pk(s, d);
    }
}

// y = s * (1/sqrt(k)) with the constant split as c_hi + c_lo (both fp32, from
// the fp64 value): the fused form rounds once, so y is the fp32 nearest to
// s * c except when s * c is within ~2^-47 relative of a rounding midpoint.
template <int N>
__device__ __forceinline__ void normalize(f32x2 (&p)[N / 2], float c_hi, float c_lo)
{
    const f32x2 hi = pk(c_hi, c_hi), lo = pk(c_lo, c_lo);
#pragma unroll
    for (int k = 0; k < N / 2; ++k) p[k] = fma2(p[k], hi, mul2(p[k], lo));
}

// ---------------------------------------------------------------- warp helpers
template <int LANES>
__device__ __forceinline__ float group_max(float m)
{
#pragma unroll
    for (int d = 1; d < LANES; d <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
    return m;
}

}  // namespace fp4q
