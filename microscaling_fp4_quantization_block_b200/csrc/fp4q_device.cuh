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

__device__ __forceinline__ void stg64(void* p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

// ---------------------------------------------------------------- async copies into shared memory
// 16-byte global -> shared copy (L2 only, no L1); src_bytes 0 writes zeros and
// reads nothing.  Completion is tracked per thread with commit / wait groups.
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr), "l"(gptr), "r"(src_bytes)
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

// Approximate reciprocal (at most 1 ulp from 1/s for normal s with a normal
// reciprocal); only used where a bound, not the rounded value, matters.
__device__ __forceinline__ float rcp_approx(float s)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
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

// Exact UE4M3 code of fp32(m / d): the fallback of the bracketed scale rule,
// kept out of line so the common path carries none of its instructions.
static __device__ __noinline__ uint32_t ue4m3_code_of_quotient(float m, float d)
{
    return ue4m3_encode(__fdiv_rn(m, d));
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

// ---------------------------------------------------------------- block scale
// Quotients that decide a code are bracketed instead of divided.  With an
// approximate reciprocal R of a divisor d (at most 1 ulp off) and
// R_lo = fp32(R (1 - 2^-19)), R_hi = fp32(R (1 + 2^-19)), the correctly rounded
// quotient q* = fp32(a / d) lies strictly between fp32(a R_lo) and fp32(a R_hi)
// for every fp32 a (the worst-case rounding errors add up to 6 units of 2^-24
// against a bracket half-width of 32 units).  Rounding to E2M1 or to UE4M3 is
// monotone in |q| and keeps the sign, so when both ends round to the same code
// that code is the code of q*; otherwise the code is recomputed from the
// correctly rounded division.  d and 1/d must both be normal floats.
constexpr float kBracketLo = 0.99999809265136719f;   // 1 - 2^-19, exact in fp32
constexpr float kBracketHi = 1.00000190734863281f;                           // 1 + 2^-19, exact in fp32

__device__ __forceinline__ bool divisor_safe(float d)
{
    const uint32_t e = as_u32(d) >> 23;            // d > 0: biased exponent
    return e >= 1u && e <= 252u;                   // d and 1/d normal
}

// Per-tensor constants of the UE scale rule.
struct ScaleConsts {
    float G;                 // per-tensor scale
    float denom;             // fp32(6 G)
    float rd_lo, rd_hi;      // bracket of 1/denom
    bool denom_ok;
};

__device__ __forceinline__ ScaleConsts scale_consts(float G)
{
    ScaleConsts c;
    c.G = G;
    c.denom = __fmul_rn(6.0f, G);
    c.denom_ok = divisor_safe(c.denom);
    const float r = rcp_approx(c.denom);
    c.rd_lo = __fmul_rn(r, kBracketLo);
    c.rd_hi = __fmul_rn(r, kBracketHi);
    return c;
}

// UE4M3 scales of two blocks at once (block maxima m0, m1): codes, block
// scales S = fp32(decode(code) G) and the brackets [r_lo, r_hi] of 1/S (both 0
// for a zero block).  Returns false when some 1/S cannot be bracketed (S or
// 1/S not a normal float), i.e. when elements must be divided.
__device__ __forceinline__ bool block_scale_ue4m3_pair(float m0, float m1, const ScaleConsts& k, uint32_t& c0,
                                                       uint32_t& c1, float& S0, float& S1, float& rlo0, float& rlo1,
                                                       float& rhi0, float& rhi1)
{
    const f32x2 mm = pk(m0, m1);
    float l0, l1, h0, h1;
    upk(mul2(mm, pk(k.rd_lo, k.rd_lo)), l0, l1);
    upk(mul2(mm, pk(k.rd_hi, k.rd_hi)), h0, h1);
    uint32_t codes = ue4m3_encode2(l0, l1);                    // low byte: block 0
    if (codes != ue4m3_encode2(h0, h1) || !k.denom_ok)         // rare: a quotient at a rounding tie
        codes = ue4m3_code_of_quotient(m0, k.denom) | (ue4m3_code_of_quotient(m1, k.denom) << 8);
    c0 = codes & 0xffu;
    c1 = codes >> 8;
    float d0, d1;
    ue4m3_decode2_hw(codes, d0, d1);
    upk(mul2(pk(d0, d1), pk(k.G, k.G)), S0, S1);
    const f32x2 r = pk(rcp_approx(S0), rcp_approx(S1));
    float a0, a1, b0, b1;
    upk(mul2(r, pk(kBracketLo, kBracketLo)), a0, a1);
    upk(mul2(r, pk(kBracketHi, kBracketHi)), b0, b1);
    rlo0 = S0 == 0.0f ? 0.0f : a0;                             // zero-rounded block
    rhi0 = S0 == 0.0f ? 0.0f : b0;
    rlo1 = S1 == 0.0f ? 0.0f : a1;
    rhi1 = S1 == 0.0f ? 0.0f : b1;
    return (S0 == 0.0f || divisor_safe(S0)) && (S1 == 0.0f || divisor_safe(S1));
}

// Scale byte of a block with absolute maximum m ("max" rule), the block's
// dequantization scale S and the bracket [r_lo, r_hi] of 1/S (0 for a zero
// block; `exact` false when 1/S cannot be bracketed and elements must divide).
//   E8M0:  S = 2^(floor(log2 m) - 2), r_lo = r_hi = 1/S exactly.
//   UE4M3: the paired routine above on (m, m).
//   UE5M3: s = code nearest fp32(m / denom) (exact division), S = fp32(decode(s) G).
template <int FMT>
__device__ __forceinline__ uint32_t block_scale(float m, const ScaleConsts& k, float& S, float& r_lo,
                                                float& r_hi, bool& exact)
{
    uint32_t c;
    if constexpr (FMT == kE8M0) {
        c = e8m0_from_amax(m);
        S = e8m0_decode(c);
        r_lo = r_hi = e8m0_inverse(c);
        exact = true;
        return c;
    } else if constexpr (FMT == kUE4M3) {
        uint32_t c1;
        float S1, a1, b1;
        exact = block_scale_ue4m3_pair(m, m, k, c, c1, S, S1, r_lo, a1, r_hi, b1);
        return c;
    } else {
        c = ue5m3_encode(__fdiv_rn(m, k.denom));
        S = __fmul_rn(ue5m3_decode(c), k.G);
        if (S == 0.0f) {
            r_lo = r_hi = 0.0f;
            exact = true;
        } else {
            const float r = rcp_approx(S);
            upk(mul2(pk(r, r), pk(kBracketLo, kBracketHi)), r_lo, r_hi);
            exact = divisor_safe(S);
        }
        return c;
    }
}

// ---------------------------------------------------------------- Hadamard
// Values are held as N/2 fp32 pairs p[k] = (v[2k], v[2k+1]).  In-register
// Sylvester Hadamard transform of every run of CH consecutive values (natural
// order: y_i = sum_j (-1)^popcount(i & j) x_j): the distance-1 stage mixes the
// two halves of each pair, the others combine whole pairs.
template <int N, int CH>
__device__ __forceinline__ void fwht_inreg(f32x2 (&p)[N / 2])
{
    if constexpr (CH >= 2) {
#pragma unroll
        for (int k = 0; k < N / 2; ++k) {
            float a, b;
            upk(p[k], a, b);
            p[k] = pk(__fadd_rn(a, b), __fsub_rn(a, b));
        }
    }
#pragma unroll
    for (int h = 2; h < CH; h <<= 1) {
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

// Butterfly stages across LANES consecutive lanes (each lane holding the next
// N values of the run): lane bit d pairs lane l with l ^ d; the lower lane
// keeps a + b, the upper one a - b, a being the lower lane's value; both are
// other + sign * own with sign = +1 / -1.
template <int N, int LANES>
__device__ __forceinline__ void fwht_xlane(f32x2 (&p)[N / 2], int lane)
{
#pragma unroll
    for (int d = 1; d < LANES; d <<= 1) {
        const float sg = (lane & d) ? -1.0f : 1.0f;
        const f32x2 sg2 = pk(sg, sg);
#pragma unroll
        for (int k = 0; k < N / 2; ++k) {
            float a, b;
            upk(p[k], a, b);
            const f32x2 other = pk(__shfl_xor_sync(0xffffffffu, a, d), __shfl_xor_sync(0xffffffffu, b, d));
            p[k] = fma2(p[k], sg2, other);            // exact: sign * own is exact
        }
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
