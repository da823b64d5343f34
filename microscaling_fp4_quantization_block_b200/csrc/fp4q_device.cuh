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

__device__ __forceinline__ void stg64(void* p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
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

__device__ __forceinline__ float ue4m3_decode(uint32_t c)
{
    uint32_t e = c >> 3, m = c & 7u;
    if (c >= 0x7fu) return as_f32(0x7fc00000u);
    if (e == 0u) return __fmul_rn((float)m, 0.001953125f);          // m * 2^-9, exact
    return as_f32(((e + 120u) << 23) | (m << 20));
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

// ---------------------------------------------------------------- block scale
// Per-block scale of the "max" rule.  Returns the scale byte and sets S (the
// dequantization scale, fp32) and R (1/S for the quantizer's product).
//   E8M0:          S = 2^(floor(log2 m)-2), R exact.
//   UE4M3 / UE5M3: s = code nearest fp32(m / denom) (denom = fp32(6 G)),
//                  S = fp32(decode(s) * G), R = correctly rounded 1/S.
template <int FMT>
__device__ __forceinline__ uint32_t block_scale(float m, float G, float denom, float& S, float& R)
{
    if constexpr (FMT == kE8M0) {
        uint32_t c = e8m0_from_amax(m);
        S = e8m0_decode(c);
        R = e8m0_inverse(c);
        return c;
    } else {
        float sf = __fdiv_rn(m, denom);
        uint32_t c = (FMT == kUE4M3) ? ue4m3_encode(sf) : ue5m3_encode(sf);
        float d = (FMT == kUE4M3) ? ue4m3_decode(c) : ue5m3_decode(c);
        S = __fmul_rn(d, G);
        R = __frcp_rn(S);
        return c;
    }
}

// For the UE formats the quotient y/S is first taken as q0 = fp32(y * R) with
// R = fp32(1/S) correctly rounded (S and 1/S normal).  Then
// |y*R - y/S| <= 2^-24 |y/S| and |q0 - y/S| < 2 ulp(y/S) <= 2^-22 |y/S|, so the
// correctly rounded quotient q* = fp32(y/S) lies strictly inside
// [fp32(q0 (1 - 2^-20)), fp32(q0 (1 + 2^-20))].  E2M1 rounding is monotone in
// |q| and keeps the sign, so when the two ends round to the same code, that
// code is the code of q*; otherwise the element is recomputed with a
// correctly rounded division.
constexpr float kBracketLo = 0.99999904632568359375f;   // 1 - 2^-20, exact in fp32
constexpr float kBracketHi = 1.00000095367431640625f;   // 1 + 2^-20, exact in fp32

// S is usable for the reciprocal product when S and 1/S are both normal.
__device__ __forceinline__ bool scale_product_safe(float S)
{
    uint32_t e = as_u32(S) >> 23;
    return e >= 1u && e <= 252u;
}

// ---------------------------------------------------------------- Hadamard
// In-register Sylvester Hadamard transform of every run of CH consecutive
// values of v[N] (natural order: y_i = sum_j (-1)^popcount(i&j) x_j).
template <int N, int CH>
__device__ __forceinline__ void fwht_inreg(float (&v)[N])
{
#pragma unroll
    for (int h = 1; h < CH; h <<= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
        }
    }
}

// Butterfly stages across LANES consecutive lanes (each lane holding the next
// N values of the run): lane bit p pairs lane l with l ^ 2^p; the lower lane
// keeps a + b, the upper one a - b, where a is the lower lane's value.
template <int N, int LANES>
__device__ __forceinline__ void fwht_xlane(float (&v)[N], int lane)
{
#pragma unroll
    for (int d = 1; d < LANES; d <<= 1) {
        const bool upper = (lane & d) != 0;
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float other = __shfl_xor_sync(0xffffffffu, v[i], d);
            v[i] = upper ? __fsub_rn(other, v[i]) : __fadd_rn(v[i], other);
        }
    }
}

// y = s * (1/sqrt(k)) with the constant split as c_hi + c_lo (both fp32, from
// the fp64 value): the fused form rounds once, so y is the fp32 nearest to
// s * c except when s * c is within ~2^-47 relative of a rounding midpoint.
template <int N>
__device__ __forceinline__ void normalize(float (&v)[N], float c_hi, float c_lo)
{
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = __fmaf_rn(v[i], c_hi, __fmul_rn(v[i], c_lo));
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
