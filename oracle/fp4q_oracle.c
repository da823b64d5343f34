/*
 * fp4q_oracle.c -- plain, slow, single-threaded CPU oracle for block-wise
 * microscaling FP4 quantization (MXFP4, NVFP4 and the UE4M3 block-size sweep).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product library
 * (libfp4q.so) shares no code, header, table or constant with this file, and
 * neither one includes or calls the other.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (no -ffast-math, no FMA
 * contraction, so every float operation below is one IEEE-754 binary32
 * operation rounded to nearest-even, exactly as written).
 *
 * Sources (page title, section):
 *  [D]  "Diagnosing FP4 inference: a layer-wise and block-wise sensitivity
 *       analysis of NVFP4 and MXFP4", technical summary, Methodology: MXFP4 =
 *       blocks of 32 E2M1 elements sharing an 8-bit exponent; NVFP4 = blocks of
 *       16 with a scale and "max" calibration; weights kept in 16 bits,
 *       quantized on the fly and dequantized for the compute.
 *  [B]  "Bridging the Gap Between Promise and Performance for Microscaling FP4
 *       Quantization", technical summary s1-s3: MXFP4 scales are powers of two
 *       (E8M0), NVFP4 scales are E4M3; round-to-nearest (RTN) is the baseline
 *       quantizer; block-wise Hadamard rotations of weights and activations.
 *  [F]  "Finer is better? Limits of micro-scaling formats in LLMs", Theoretical
 *       framework and Contributions: unsigned E4M3 (UE4M3) scales with minimum
 *       non-zero value 2^-9; UE4M3 under a per-tensor scale (UE4M3-S); the
 *       proposed UE5M3 scale with minimum 2^-17; MSE per block and per tensor,
 *       split into non-max elements, block max and zero-rounded blocks.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - E2M1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}; round to nearest, ties to the
 *    even code, saturating at 6; the sign bit is kept, so a negative value
 *    that rounds to zero is code 0x8.
 *  - MX scale: 2^(floor(log2 amax) - 2) (2 = largest E2M1 exponent), stored
 *    as the E8M0 byte e+127, e clamped to [-127, 127]; amax = 0 gives byte 0.
 *  - NV scale: s = UE4M3_RNE_satfinite( fp32(amax / fp32(6*G)) ), block scale
 *    S = fp32(decode(s) * G); G = 1 without a per-tensor scale, otherwise
 *    G = fp32(amax_tensor / 2688) (2688 = 6 * 448), or 1 if amax_tensor = 0.
 *  - A block whose S is 0 is zero-rounded and stores all-zero nibbles.
 *    Otherwise nibble = E2M1(fp32(y / S)) with correctly rounded division.
 *  - Blocks are b consecutive elements of a row; rotations act on k
 *    consecutive elements of a row, y = H_k x / sqrt(k), H_k the Sylvester
 *    Hadamard matrix H[i][j] = (-1)^popcount(i & j), evaluated densely in fp64
 *    and rounded once to fp32.
 *  - Packing: byte j of the code stream holds element 2j in its low nibble and
 *    element 2j+1 in its high nibble; scale bytes are row-major [rows][cols/b].
 *  - MSE is measured in the domain that was quantized (the rotated one when a
 *    rotation is applied); errors and sums are fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_VERSION 1

enum { ORC_E8M0 = 0, ORC_UE4M3 = 1, ORC_UE5M3 = 2 };
enum { ORC_G_NONE = 0, ORC_G_COMPUTE = 1, ORC_G_GIVEN = 2 };
enum { ORC_OK = 0, ORC_EARG = -1, ORC_ESHAPE = -2, ORC_ENOMEM = -3 };

int orc_version(void) { return ORC_VERSION; }

/* ------------------------------------------------------------------------ */
/* bit views                                                                 */

static float f32_of_bits(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t bits_of_f32(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

/* bf16 -> fp32 is exact: the bf16 pattern is the top half of the fp32 one. */
float orc_bf16_to_f32(uint16_t h) { return f32_of_bits((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t b = bits_of_f32(f);
    if ((b & 0x7f800000u) == 0x7f800000u && (b & 0x007fffffu))
        return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t keep = b >> 16;
    uint32_t rest = b & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u)))
        keep += 1u;
    return (uint16_t)keep;
}

void orc_f32_to_bf16_array(const float* in, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(in[i]);
}

void orc_bf16_to_f32_array(const uint16_t* in, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(in[i]);
}

/* ------------------------------------------------------------------------ */
/* E2M1 element format [D] Methodology ("E2M1"), [B] s1.                     */
/* Magnitude of each 3-bit code: 1 exponent-2-bit, 1 mantissa-bit float with */
/* bias 1; code 1 is the subnormal 0.5.                                      */

static const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float orc_e2m1_decode(uint8_t nibble)
{
    double v = kE2M1Mag[nibble & 7u];
    return (float)((nibble & 8u) ? -v : v);
}

/* Round-to-nearest (RTN, [B] s1) onto the E2M1 grid: the grid point closest
 * to |r|; on an exact tie the even code wins; beyond 6 the result saturates
 * to 6.  The sign of r (including the sign of zero) is kept in bit 3. */
uint8_t orc_e2m1_encode(float r)
{
    uint8_t sign = signbit(r) ? 8u : 0u;
    double a = fabs((double)r);
    if (a > 6.0) return (uint8_t)(sign | 7u);      /* saturate (and +inf) */
    int best = 0;
    double bestd = a;                              /* distance to 0 */
    for (int i = 1; i < 8; ++i) {
        double d = fabs(a - kE2M1Mag[i]);          /* exact in fp64 */
        if (d < bestd || (d == bestd && (i & 1) == 0)) {
            best = i;
            bestd = d;
        }
    }
    return (uint8_t)(sign | (uint8_t)best);
}

/* ------------------------------------------------------------------------ */
/* E8M0 shared exponent [D] Methodology, [B] s1-s2 (power-of-two scales).    */

float orc_e8m0_decode(uint8_t c)
{
    if (c == 0xffu) return f32_of_bits(0x7fc00000u);
    return ldexpf(1.0f, (int)c - 127);             /* c = 0 gives 2^-127 */
}

/* Scale exponent for a block with absolute maximum m: floor(log2 m) minus the
 * largest E2M1 exponent (2), clamped to the E8M0 range; m = 0 gives byte 0. */
uint8_t orc_e8m0_from_amax(float m)
{
    if (!isfinite(m)) return 0xffu;
    if (m == 0.0f) return 0u;
    int ex;
    (void)frexp((double)m, &ex);                   /* m = f * 2^ex, f in [0.5,1) */
    int e = (ex - 1) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return (uint8_t)(e + 127);
}

/* ------------------------------------------------------------------------ */
/* UE4M3 block scale [B] s1 (E4M3), [F] Theoretical framework (unsigned      */
/* E4M3, smallest non-zero value 2^-9).  Bias 7, 4 exponent and 3 mantissa   */
/* bits; code 0x7F is NaN, so the largest finite value is 0x7E = 448.        */

float orc_ue4m3_decode(uint8_t c)
{
    if (c >= 0x7fu) return f32_of_bits(0x7fc00000u);
    int e = c >> 3, m = c & 7;
    if (e == 0) return (float)ldexp((double)m, -9);
    return (float)ldexp((double)(8 + m), e - 10);
}

/* Nearest finite UE4M3 value to s >= 0 (ties to the even code), with
 * saturation to 448: a bisection over the monotone value table. */
static uint8_t nearest_code_in_table(double s, float (*dec)(uint8_t), int last)
{
    if (s >= (double)dec((uint8_t)last)) return (uint8_t)last;
    int lo = 0, hi = last;                         /* dec(lo) <= s < dec(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if ((double)dec((uint8_t)mid) <= s) lo = mid; else hi = mid;
    }
    double dlo = s - (double)dec((uint8_t)lo);
    double dhi = (double)dec((uint8_t)hi) - s;
    if (dlo < dhi) return (uint8_t)lo;
    if (dhi < dlo) return (uint8_t)hi;
    return (uint8_t)((lo & 1) ? hi : lo);
}

uint8_t orc_ue4m3_encode(float s)
{
    if (isnan(s)) return 0x7fu;
    if (s <= 0.0f) return 0u;
    return nearest_code_in_table((double)s, orc_ue4m3_decode, 0x7e);
}

/* ------------------------------------------------------------------------ */
/* UE5M3 block scale [F] Contributions: the unused sign bit of UE4M3 becomes */
/* a fifth exponent bit, lowering the smallest non-zero value to 2^-17,      */
/* which fixes the bias at 15.  The pages give no maximum or NaN code; the   */
/* reading here follows E4M3: only 0xFF is NaN, so 0xFE = 1.75*2^16 = 114688 */
/* is the largest finite value.                                              */

float orc_ue5m3_decode(uint8_t c)
{
    if (c == 0xffu) return f32_of_bits(0x7fc00000u);
    int e = c >> 3, m = c & 7;
    if (e == 0) return (float)ldexp((double)m, -17);
    return (float)ldexp((double)(8 + m), e - 18);
}

uint8_t orc_ue5m3_encode(float s)
{
    if (isnan(s)) return 0xffu;
    if (s <= 0.0f) return 0u;
    return nearest_code_in_table((double)s, orc_ue5m3_decode, 0xfe);
}

/* Array forms used by the exhaustive codec tests: encode every fp32 whose bit
 * pattern lies in [lo, lo + count). */
void orc_e2m1_encode_bits_range(uint32_t lo, uint64_t count, uint8_t* out)
{
    for (uint64_t i = 0; i < count; ++i) out[i] = orc_e2m1_encode(f32_of_bits(lo + (uint32_t)i));
}

void orc_ue4m3_encode_bits_range(uint32_t lo, uint64_t count, uint8_t* out)
{
    for (uint64_t i = 0; i < count; ++i) out[i] = orc_ue4m3_encode(f32_of_bits(lo + (uint32_t)i));
}

void orc_e2m1_encode_array(const float* r, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(r[i]);
}

void orc_ue4m3_encode_array(const float* s, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_ue4m3_encode(s[i]);
}

void orc_ue5m3_encode_array(const float* s, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_ue5m3_encode(s[i]);
}

/* ------------------------------------------------------------------------ */
/* Block-wise Hadamard micro-rotation [B] s2 and s3.1: each run of k          */
/* consecutive elements of a row is replaced by H_k x / sqrt(k).             */

static int popcount_u32(uint32_t v)
{
    int c = 0;
    while (v) { c += (int)(v & 1u); v >>= 1; }
    return c;
}

int orc_hadamard(const float* x, int64_t n, int k, float* y)
{
    if (k <= 0 || (k & (k - 1)) != 0 || n % k != 0) return ORC_EARG;
    const double norm = 1.0 / sqrt((double)k);
    for (int64_t base = 0; base < n; base += k) {
        for (int i = 0; i < k; ++i) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                double h = (popcount_u32((uint32_t)(i & j)) & 1) ? -1.0 : 1.0;
                acc += h * (double)x[base + j];
            }
            y[base + i] = (float)(acc * norm);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Argument checks shared by the entry points below.                          */

static int is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

static int check_layout(int64_t rows, int64_t cols, int fmt, int block, int rot)
{
    if (rows < 0 || cols < 0) return ORC_ESHAPE;
    if (fmt != ORC_E8M0 && fmt != ORC_UE4M3 && fmt != ORC_UE5M3) return ORC_EARG;
    if (!is_pow2(block) || block < 8 || block > 256) return ORC_EARG;
    if (cols % block) return ORC_ESHAPE;
    if (rot != 0) {
        if (!is_pow2(rot) || rot < 2) return ORC_EARG;
        if (cols % rot) return ORC_ESHAPE;
    }
    return ORC_OK;
}

/* Rotated (or plain) fp32 view of the input, allocated by the caller of this
 * helper and freed by it. */
static float* domain_values(const float* x, int64_t n, int rot)
{
    float* y = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!y) return NULL;
    if (rot) orc_hadamard(x, n, rot, y);
    else if (n) memcpy(y, x, (size_t)n * sizeof(float));
    return y;
}

/* Largest |y| over a whole tensor: the "max" calibration of the per-tensor
 * scale ([F] Results: UE4M3 with a dynamic per-tensor scale). */
float orc_tensor_amax(const float* y, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(y[i]);
        if (a > m) m = a;
    }
    return m;
}

/* Per-tensor scale from the tensor's absolute maximum: G = amax / (6 * 448),
 * the largest E2M1 value times the largest UE4M3 value, so that the largest
 * block of the tensor gets a UE4M3 scale near 448. */
float orc_global_scale_from_amax(float amax)
{
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;
}

/* Block scale S (fp32) and the stored scale byte for a block with absolute
 * maximum m ("max" calibration, [D] Methodology). */
static float block_scale(int fmt, float m, float G, uint8_t* code)
{
    if (fmt == ORC_E8M0) {
        *code = orc_e8m0_from_amax(m);
        return orc_e8m0_decode(*code);
    }
    float denom = 6.0f * G;
    float sf = m / denom;
    if (fmt == ORC_UE4M3) {
        *code = orc_ue4m3_encode(sf);
        return (float)((double)orc_ue4m3_decode(*code) * (double)G);
    }
    *code = orc_ue5m3_encode(sf);
    return (float)((double)orc_ue5m3_decode(*code) * (double)G);
}

static float scale_of_code(int fmt, uint8_t code, float G)
{
    if (fmt == ORC_E8M0) return orc_e8m0_decode(code);
    if (fmt == ORC_UE4M3) return (float)((double)orc_ue4m3_decode(code) * (double)G);
    return (float)((double)orc_ue5m3_decode(code) * (double)G);
}

/* ------------------------------------------------------------------------ */
/* Quantization: optional rotation, per-block absmax, scale rule, RTN onto    */
/* E2M1, 4-bit packing with one scale byte per block ([D] Methodology,       */
/* [B] s1-s3, [F] Theoretical framework).                                    */

int orc_quantize_f32(const float* x, int64_t rows, int64_t cols, int fmt, int block,
                     int rot, int gmode, float* gscale, uint8_t* codes, uint8_t* scales)
{
    int st = check_layout(rows, cols, fmt, block, rot);
    if (st) return st;
    if (fmt == ORC_E8M0 && gmode != ORC_G_NONE) return ORC_EARG;
    if (gmode != ORC_G_NONE && gmode != ORC_G_COMPUTE && gmode != ORC_G_GIVEN) return ORC_EARG;
    if (gmode != ORC_G_NONE && !gscale) return ORC_EARG;
    const int64_t n = rows * cols;
    float* y = domain_values(x, n, rot);
    if (!y) return ORC_ENOMEM;

    float G = 1.0f;
    if (gmode == ORC_G_COMPUTE) {
        G = orc_global_scale_from_amax(orc_tensor_amax(y, n));
        *gscale = G;
    } else if (gmode == ORC_G_GIVEN) {
        G = *gscale;
    }

    memset(codes, 0, (size_t)(n / 2));
    for (int64_t b0 = 0, bi = 0; b0 < n; b0 += block, ++bi) {
        float m = 0.0f;
        for (int i = 0; i < block; ++i) {
            float a = fabsf(y[b0 + i]);
            if (a > m) m = a;
        }
        uint8_t sc;
        float S = block_scale(fmt, m, G, &sc);
        scales[bi] = sc;
        for (int i = 0; i < block; ++i) {
            uint8_t nib = 0u;
            if (S != 0.0f) nib = orc_e2m1_encode(y[b0 + i] / S);
            int64_t e = b0 + i;
            codes[e >> 1] |= (uint8_t)(nib << ((e & 1) ? 4 : 0));
        }
    }
    free(y);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* MSE-optimised block scales ([B] s3, MR-GPTQ item 2, "MSE-optimised grids": */
/* each block's scale is chosen to minimise its squared reconstruction error  */
/* instead of by the max rule).  The pages give no search procedure; the     */
/* reading taken here: the candidates are the max-rule code s0 and its        */
/* neighbours in code order, tried as s0, s0+1 .. s0+above, s0-1 .. s0-below */
/* (codes outside the format's finite range are skipped); a candidate         */
/* replaces the best so far only when its error is strictly smaller, so ties  */
/* keep the earlier one and the max rule wins any tie.  The error of a scale  */
/* S is sum_i (y_i - v_i)^2 with v_i = fp32(decode(E2M1(y_i / S)) S), and    */
/* v_i = 0 when S = 0 (a zero-rounded block).  The pages fix no precision, so */
/* the criterion is the exact error: each d_i = y_i - v_i is exact in fp64,   */
/* its square is exact (24-bit significands), and the fp64 sum of b <= 256    */
/* such terms is within 2^-45 relative of the true sum.                       */

static int last_finite_code(int fmt)
{
    if (fmt == ORC_E8M0) return 0xfe;
    if (fmt == ORC_UE4M3) return 0x7e;
    return 0xfe;
}

static double block_sq_error(const float* y, int block, float S)
{
    double sum = 0.0;
    for (int i = 0; i < block; ++i) {
        float v = 0.0f;
        if (S != 0.0f) v = (float)((double)orc_e2m1_decode(orc_e2m1_encode(y[i] / S)) * (double)S);
        double d = (double)y[i] - (double)v;
        sum += d * d;
    }
    return sum;
}

int orc_quantize_search_f32(const float* x, int64_t rows, int64_t cols, int fmt, int block,
                            int rot, int gmode, int below, int above, float* gscale,
                            uint8_t* codes, uint8_t* scales)
{
    if (below < 0 || below > 16 || above < 0 || above > 16) return ORC_EARG;
    /* the max rule first: its scales are the search's starting codes */
    int st = orc_quantize_f32(x, rows, cols, fmt, block, rot, gmode, gscale, codes, scales);
    if (st) return st;
    const int64_t n = rows * cols;
    float* y = domain_values(x, n, rot);
    if (!y) return ORC_ENOMEM;
    const float G = gmode != ORC_G_NONE ? *gscale : 1.0f;
    const int last = last_finite_code(fmt);

    memset(codes, 0, (size_t)(n / 2));
    for (int64_t b0 = 0, bi = 0; b0 < n; b0 += block, ++bi) {
        const int s0 = scales[bi];
        int best = s0;
        double best_err = block_sq_error(y + b0, block, scale_of_code(fmt, (uint8_t)s0, G));
        for (int j = 1; j <= above + below; ++j) {
            const int c = j <= above ? s0 + j : s0 - (j - above);
            if (c < 0 || c > last) continue;
            double err = block_sq_error(y + b0, block, scale_of_code(fmt, (uint8_t)c, G));
            if (err < best_err) {
                best = c;
                best_err = err;
            }
        }
        scales[bi] = (uint8_t)best;
        const float S = scale_of_code(fmt, (uint8_t)best, G);
        for (int i = 0; i < block; ++i) {
            uint8_t nib = 0u;
            if (S != 0.0f) nib = orc_e2m1_encode(y[b0 + i] / S);
            int64_t e = b0 + i;
            codes[e >> 1] |= (uint8_t)(nib << ((e & 1) ? 4 : 0));
        }
    }
    free(y);
    return ORC_OK;
}

int orc_quantize_search_bf16(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int block,
                             int rot, int gmode, int below, int above, float* gscale,
                             uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || cols < 0) return ORC_ESHAPE;
    const int64_t n = rows * cols;
    float* xf = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!xf) return ORC_ENOMEM;
    orc_bf16_to_f32_array(x, n, xf);
    int st = orc_quantize_search_f32(xf, rows, cols, fmt, block, rot, gmode, below, above, gscale,
                                     codes, scales);
    free(xf);
    return st;
}

/* Codes for given scale bytes: every block quantized with S = decode(scale)
 * (times G for the UE formats) exactly as the max rule's blocks are. */
int orc_quantize_with_scales_f32(const float* x, int64_t rows, int64_t cols, int fmt, int block,
                                 int rot, const uint8_t* scales, float G, uint8_t* codes)
{
    int st = check_layout(rows, cols, fmt, block, rot);
    if (st) return st;
    const int64_t n = rows * cols;
    float* y = domain_values(x, n, rot);
    if (!y) return ORC_ENOMEM;
    memset(codes, 0, (size_t)(n / 2));
    for (int64_t b0 = 0, bi = 0; b0 < n; b0 += block, ++bi) {
        const float S = scale_of_code(fmt, scales[bi], G);
        for (int i = 0; i < block; ++i) {
            uint8_t nib = 0u;
            if (S != 0.0f) nib = orc_e2m1_encode(y[b0 + i] / S);
            int64_t e = b0 + i;
            codes[e >> 1] |= (uint8_t)(nib << ((e & 1) ? 4 : 0));
        }
    }
    free(y);
    return ORC_OK;
}

int orc_quantize_with_scales_bf16(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int block,
                                  int rot, const uint8_t* scales, float G, uint8_t* codes)
{
    if (rows < 0 || cols < 0) return ORC_ESHAPE;
    const int64_t n = rows * cols;
    float* xf = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!xf) return ORC_ENOMEM;
    orc_bf16_to_f32_array(x, n, xf);
    int st = orc_quantize_with_scales_f32(xf, rows, cols, fmt, block, rot, scales, G, codes);
    free(xf);
    return st;
}

int orc_quantize_bf16(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int block,
                      int rot, int gmode, float* gscale, uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || cols < 0) return ORC_ESHAPE;
    const int64_t n = rows * cols;
    float* xf = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!xf) return ORC_ENOMEM;
    orc_bf16_to_f32_array(x, n, xf);
    int st = orc_quantize_f32(xf, rows, cols, fmt, block, rot, gmode, gscale, codes, scales);
    free(xf);
    return st;
}

/* ------------------------------------------------------------------------ */
/* Dequantization ([D] Methodology: quantized on the fly, then dequantized   */
/* for the compute): v = fp32(decode(nibble) * S).  With rot = k the result  */
/* is rotated back (H_k / sqrt(k) is its own inverse); rot = 0 leaves it in  */
/* the quantized domain.                                                     */

int orc_dequantize(const uint8_t* codes, const uint8_t* scales, float G, int64_t rows,
                   int64_t cols, int fmt, int block, int rot, float* out)
{
    int st = check_layout(rows, cols, fmt, block, rot);
    if (st) return st;
    const int64_t n = rows * cols;
    float* v = rot ? (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float)) : out;
    if (!v) return ORC_ENOMEM;
    for (int64_t e = 0; e < n; ++e) {
        float S = scale_of_code(fmt, scales[e / block], G);
        uint8_t nib = (uint8_t)((codes[e >> 1] >> ((e & 1) ? 4 : 0)) & 0xfu);
        v[e] = (float)((double)orc_e2m1_decode(nib) * (double)S);
    }
    if (rot) {
        orc_hadamard(v, n, rot, out);
        free(v);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* MSE per block and per tensor with the three-term split of [F] Theoretical */
/* framework: (1) non-max elements, (2) the block maximum, (3) zero-rounded  */
/* blocks (every dequantized value of the block is 0).  The block maximum is */
/* the first element of largest |y|.  terms = {total, non-max, max, zero},   */
/* each a sum of squared errors divided by the element count, so the three   */
/* parts add up to the per-tensor MSE.  block_mse may be NULL.               */

int orc_block_mse_f32(const float* x, const uint8_t* codes, const uint8_t* scales, float G,
                      int64_t rows, int64_t cols, int fmt, int block, int rot,
                      double* block_mse, double* terms)
{
    int st = check_layout(rows, cols, fmt, block, rot);
    if (st) return st;
    const int64_t n = rows * cols;
    float* y = domain_values(x, n, rot);
    if (!y) return ORC_ENOMEM;
    double t_total = 0.0, t_nonmax = 0.0, t_max = 0.0, t_zero = 0.0;
    for (int64_t b0 = 0, bi = 0; b0 < n; b0 += block, ++bi) {
        float S = scale_of_code(fmt, scales[bi], G);
        int arg = 0;
        float m = -1.0f;
        int all_zero = 1;
        double sum = 0.0;
        for (int i = 0; i < block; ++i) {
            int64_t e = b0 + i;
            uint8_t nib = (uint8_t)((codes[e >> 1] >> ((e & 1) ? 4 : 0)) & 0xfu);
            float v = (float)((double)orc_e2m1_decode(nib) * (double)S);
            if (v != 0.0f) all_zero = 0;
            double d = (double)y[e] - (double)v;
            sum += d * d;
            if (fabsf(y[e]) > m) { m = fabsf(y[e]); arg = i; }
        }
        if (block_mse) block_mse[bi] = sum / (double)block;
        t_total += sum;
        if (all_zero) {
            t_zero += sum;
        } else {
            for (int i = 0; i < block; ++i) {
                int64_t e = b0 + i;
                uint8_t nib = (uint8_t)((codes[e >> 1] >> ((e & 1) ? 4 : 0)) & 0xfu);
                float v = (float)((double)orc_e2m1_decode(nib) * (double)S);
                double d = (double)y[e] - (double)v;
                if (i == arg) t_max += d * d; else t_nonmax += d * d;
            }
        }
    }
    free(y);
    double inv = n > 0 ? 1.0 / (double)n : 0.0;
    terms[0] = t_total * inv;
    terms[1] = t_nonmax * inv;
    terms[2] = t_max * inv;
    terms[3] = t_zero * inv;
    return ORC_OK;
}

int orc_block_mse_bf16(const uint16_t* x, const uint8_t* codes, const uint8_t* scales,
                       float G, int64_t rows, int64_t cols, int fmt, int block, int rot,
                       double* block_mse, double* terms)
{
    if (rows < 0 || cols < 0) return ORC_ESHAPE;
    const int64_t n = rows * cols;
    float* xf = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!xf) return ORC_ENOMEM;
    orc_bf16_to_f32_array(x, n, xf);
    int st = orc_block_mse_f32(xf, codes, scales, G, rows, cols, fmt, block, rot, block_mse, terms);
    free(xf);
    return st;
}

/* ------------------------------------------------------------------------ */
/* Activation outlier statistics ([D] Methodology and Results C: the Max and  */
/* the 99.9th percentile of the activations, and their ratio, per            */
/* projection).  The pages define neither the percentile nor whether signs    */
/* count; the reading taken here: statistics of the magnitudes |x|, and the  */
/* p-quantile by nearest rank: with the magnitudes sorted ascending,          */
/* a_1 <= ... <= a_N, it is a_k for k = ceil(p N) (p N in fp64, k clamped to  */
/* [1, N]), a value that occurs in the tensor.  Per-channel maxima are the    */
/* largest |x| of each column of the [rows][cols] = [tokens][channels]        */
/* matrix.                                                                    */

static int cmp_float_asc(const void* a, const void* b)
{
    float x = *(const float*)a, y = *(const float*)b;
    return (x > y) - (x < y);
}

int64_t orc_nearest_rank(double p, int64_t n)
{
    if (n <= 0) return 0;
    double t = ceil(p * (double)n);
    int64_t k = (int64_t)t;
    if (k < 1) k = 1;
    if (k > n) k = n;
    return k;
}

int orc_outlier_stats_bf16(const uint16_t* x, int64_t rows, int64_t cols, double p, float* stats,
                           float* col_absmax)
{
    if (rows < 0 || cols < 0) return ORC_ESHAPE;
    if (!(p > 0.0 && p <= 1.0) || !stats) return ORC_EARG;
    const int64_t n = rows * cols;
    if (col_absmax)
        for (int64_t c = 0; c < cols; ++c) col_absmax[c] = 0.0f;
    if (n == 0) {
        stats[0] = 0.0f;
        stats[1] = 0.0f;
        return ORC_OK;
    }
    float* a = (float*)malloc((size_t)n * sizeof(float));
    if (!a) return ORC_ENOMEM;
    for (int64_t i = 0; i < n; ++i) {
        a[i] = fabsf(orc_bf16_to_f32(x[i]));
        if (col_absmax && a[i] > col_absmax[i % cols]) col_absmax[i % cols] = a[i];
    }
    qsort(a, (size_t)n, sizeof(float), cmp_float_asc);
    stats[0] = a[n - 1];
    stats[1] = a[orc_nearest_rank(p, n) - 1];
    free(a);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* FP4 GEMM consumer ([B] s3-4: the QuTLASS kernels take the FP4 codes and   */
/* block scales of both operands; [D] Methodology: weights are quantized on  */
/* the fly and dequantized for the compute).  The pages give no formula; the */
/* reading taken here is the exact product of the two quantized operands:    */
/*   Y[m][n] = G_A G_B sum_k q_A[m][k] s_A[m][k/b] q_B[n][k] s_B[n][k/b],     */
/* with q the E2M1 value of a nibble and s the decoded scale byte (without   */
/* the per-tensor scale), both operands [rows][K] row-major with blocks of b */
/* along K, evaluated in fp64 in k order.                                    */

int orc_fp4_gemm(const uint8_t* codes_a, const uint8_t* scales_a, float ga, int64_t m_rows,
                 const uint8_t* codes_b, const uint8_t* scales_b, float gb, int64_t n_rows,
                 int64_t k_len, int fmt, int block, double* y)
{
    int st = check_layout(m_rows, k_len, fmt, block, 0);
    if (st) return st;
    st = check_layout(n_rows, k_len, fmt, block, 0);
    if (st) return st;
    const int64_t nb = k_len / block;
    const double g = (double)ga * (double)gb;
    for (int64_t i = 0; i < m_rows; ++i) {
        for (int64_t j = 0; j < n_rows; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < k_len; ++k) {
                const int64_t ea = i * k_len + k, eb = j * k_len + k;
                const uint8_t na = (uint8_t)((codes_a[ea >> 1] >> ((ea & 1) ? 4 : 0)) & 0xfu);
                const uint8_t nbb = (uint8_t)((codes_b[eb >> 1] >> ((eb & 1) ? 4 : 0)) & 0xfu);
                const double sa = (double)scale_of_code(fmt, scales_a[i * nb + k / block], 1.0f);
                const double sb = (double)scale_of_code(fmt, scales_b[j * nb + k / block], 1.0f);
                acc += (double)orc_e2m1_decode(na) * sa * (double)orc_e2m1_decode(nbb) * sb;
            }
            y[i * n_rows + j] = acc * g;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* MSE-optimised per-tensor scale ([B] s3.2, MR-GPTQ item 2: the global      */
/* scale is optimised together with the group scales, instead of being set  */
/* by the max rule alone).  The pages give no procedure; the reading taken   */
/* here: the candidates are G_j = fp32(G0 (16 + j) / 16), j in [-below,     */
/* above] (below <= 8, above <= 15: from half to almost twice the max-rule   */
/* scale G0 = amax / 2688, 1 for an all-zero tensor), tried in the order     */
/* j = 0, 1, -1, 2, -2, ...; under each, the block scales follow the max     */
/* rule and the error is the exact (fp64) sum of squared errors over the     */
/* whole tensor; a candidate replaces the best only when its error is        */
/* strictly smaller, so ties keep the earlier one and G0 wins every tie.     */
/* UE4M3 and UE5M3 only (E8M0 has no per-tensor scale).  Writes G* to        */
/* *gscale, the error of candidate j (divided by n) to errs[j + below], and  */
/* the codes and scale bytes under G*.                                       */

int orc_global_scale_search_f32(const float* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                                int below, int above, float* gscale, double* errs, uint8_t* codes,
                                uint8_t* scales)
{
    int st = check_layout(rows, cols, fmt, block, rot);
    if (st) return st;
    if (fmt == ORC_E8M0) return ORC_EARG;
    if (below < 0 || below > 8 || above < 0 || above > 15) return ORC_EARG;
    const int64_t n = rows * cols;
    float* y = domain_values(x, n, rot);
    if (!y) return ORC_ENOMEM;
    const float g0 = orc_global_scale_from_amax(orc_tensor_amax(y, n));
    free(y);
    uint8_t* c = (uint8_t*)malloc((size_t)(n / 2 > 0 ? n / 2 : 1));
    uint8_t* s = (uint8_t*)malloc((size_t)(n / block > 0 ? n / block : 1));
    if (!c || !s) {
        free(c);
        free(s);
        return ORC_ENOMEM;
    }
    double terms[4];
    int best = 0, have = 0;
    double best_err = 0.0;
    const int span = below > above ? below : above;
    for (int t = 0; t <= 2 * span; ++t) {
        /* t = 0, 1, 2, 3, 4 ... -> j = 0, 1, -1, 2, -2, ... */
        const int j = t == 0 ? 0 : ((t & 1) ? (t + 1) / 2 : -(t / 2));
        if (j > above || -j > below) continue;
        float G = (float)((double)g0 * (double)(16 + j) / 16.0);
        st = orc_quantize_f32(x, rows, cols, fmt, block, rot, ORC_G_GIVEN, &G, c, s);
        if (st) break;
        st = orc_block_mse_f32(x, c, s, G, rows, cols, fmt, block, rot, NULL, terms);
        if (st) break;
        errs[j + below] = terms[0];
        if (!have || terms[0] < best_err) {
            best = j;
            best_err = terms[0];
            have = 1;
        }
    }
    if (!st) {
        float G = (float)((double)g0 * (double)(16 + best) / 16.0);
        *gscale = G;
        st = orc_quantize_f32(x, rows, cols, fmt, block, rot, ORC_G_GIVEN, &G, codes, scales);
    }
    free(c);
    free(s);
    return st;
}

int orc_global_scale_search_bf16(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                                 int below, int above, float* gscale, double* errs, uint8_t* codes,
                                 uint8_t* scales)
{
    if (rows < 0 || cols < 0) return ORC_ESHAPE;
    const int64_t n = rows * cols;
    float* xf = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    if (!xf) return ORC_ENOMEM;
    orc_bf16_to_f32_array(x, n, xf);
    int st = orc_global_scale_search_f32(xf, rows, cols, fmt, block, rot, below, above, gscale, errs, codes,
                                         scales);
    free(xf);
    return st;
}
