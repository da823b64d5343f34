// Exhaustive check of the quantizer's correctly rounded quotient (div2_cr in
// fp4q_device.cuh, the remainder correction used for every element and scale
// quotient of the UE formats) against IEEE division __fdiv_rn:
//   1. every bf16 significand a (both signs) against every fp32 significand b,
//      five relative exponents (a / b from 1/16 to 8): the whole unrotated path;
//   2. fp32 a whose significands lie within 2^-10 of 1 or of 2 (where the
//      first product is furthest from the quotient), against every b;
//   3. random fp32 pairs;
//   4. a = +-0 keeps its sign.
// Prints one line per check: "<name> <cases> <mismatches>" and exits 0.
#include <cstdint>
#include <cstdio>
#include "fp4q_device.cuh"

using namespace fp4q;

__device__ unsigned long long g_count[4], g_bad[4];

__device__ __forceinline__ float q_cr(float a, float b, float R)
{
    float q0, q1;
    upk(div2_cr(pk(a, -a), pk(R, R), pk(-b, -b)), q0, q1);
    return (__float_as_uint(q0) ^ 0x80000000u) == __float_as_uint(q1) ? q0 : __uint_as_float(0x7fc00001u);
}

__device__ __forceinline__ void tally(int slot, unsigned long long n, unsigned long long bad)
{
    atomicAdd(&g_count[slot], n);
    if (bad) atomicAdd(&g_bad[slot], bad);
}

__global__ void check_bf16(int bexp)
{
    const uint32_t mb = blockIdx.x * blockDim.x + threadIdx.x;
    if (mb >= (1u << 23)) return;
    const float b = __uint_as_float(((uint32_t)(127 + bexp) << 23) | mb);
    const float R = __frcp_rn(b);
    unsigned long long bad = 0;
    for (uint32_t ma = 0; ma < 128; ++ma) {
        const float a = __uint_as_float((127u << 23) | (ma << 16));
        bad += __float_as_uint(q_cr(a, b, R)) != __float_as_uint(__fdiv_rn(a, b));
    }
    tally(0, 256, bad);          // q_cr checks a and -a together
}

__global__ void check_edges(int which)
{
    const uint32_t mb = blockIdx.x * blockDim.x + threadIdx.x;
    if (mb >= (1u << 23)) return;
    const float b = __uint_as_float((127u << 23) | mb);
    const float R = __frcp_rn(b);
    unsigned long long bad = 0;
    for (uint32_t k = 0; k < 1024; ++k) {
        const uint32_t ma = which ? (0x7fffffu - k * 8u) : (k * 8u);
        const float a = __uint_as_float((127u << 23) | ma);
        bad += __float_as_uint(q_cr(a, b, R)) != __float_as_uint(__fdiv_rn(a, b));
    }
    tally(1, 2048, bad);
}

__device__ __forceinline__ uint32_t mix(uint32_t x)
{
    x ^= x >> 16; x *= 0x7feb352du; x ^= x >> 15; x *= 0x846ca68bu; x ^= x >> 16;
    return x;
}

__global__ void check_random(uint32_t seed, int iters)
{
    const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
    unsigned long long bad = 0;
    for (int i = 0; i < iters; ++i) {
        const uint32_t u = mix(t * 2654435761u + (uint32_t)i * 97u + seed), v = mix(u ^ 0x9e3779b9u);
        const float b = __uint_as_float((u & 0x7fffffu) | ((100u + (u >> 23) % 50u) << 23));
        const float a = __uint_as_float((v & 0x7fffffu) | ((96u + (v >> 23) % 64u) << 23));
        const float R = __frcp_rn(b);
        bad += __float_as_uint(q_cr(a, b, R)) != __float_as_uint(__fdiv_rn(a, b));
    }
    tally(2, 2ull * iters, bad);
}

__global__ void check_zero()
{
    const float b = 0.7f, R = __frcp_rn(b);
    float p, m;
    upk(div2_cr(pk(0.0f, -0.0f), pk(R, R), pk(-b, -b)), p, m);
    tally(3, 2, (__float_as_uint(p) != 0u) + (__float_as_uint(m) != 0x80000000u));
}

int main()
{
    for (int e = -3; e <= 1; ++e) check_bf16<<<(1 << 23) / 256, 256>>>(e);
    check_edges<<<(1 << 23) / 256, 256>>>(0);
    check_edges<<<(1 << 23) / 256, 256>>>(1);
    check_random<<<148 * 8, 256>>>(20260101u, 4096);
    check_zero<<<1, 1>>>();
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        printf("cuda %s\n", cudaGetErrorString(e));
        return 1;
    }
    unsigned long long cnt[4], bad[4];
    cudaMemcpyFromSymbol(cnt, g_count, sizeof(cnt));
    cudaMemcpyFromSymbol(bad, g_bad, sizeof(bad));
    const char* names[4] = {"bf16_all", "fp32_edges", "fp32_random", "signed_zero"};
    for (int i = 0; i < 4; ++i) printf("%s %llu %llu\n", names[i], cnt[i], bad[i]);
    return 0;
}
