/*
 * fco.c -- CPU oracle for the low-bit two-step quantized all-reduce of
 * "Flash Communication: Reducing Tensor Parallelization Bottleneck for Fast
 * Large Language Model Inference" (sciencestack.ai/paper/2412.04964).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, scalar definition
 * that the CUDA library is checked against.  Only the tests, the smoke check
 * and the CPU-baseline leg of the benchmark may load it; the product path never
 * does.  It shares no source with the CUDA library.
 *
 * What the page fixes (TL;DR; Fig. 4; Fig. 5 right):
 *   - activations are compressed with low-bit quantization before the
 *     all-reduce, and the all-reduce is done in two steps: a reduce-scatter
 *     (RS) and an all-gather (AG);
 *   - quantization happens per block of contiguous elements along the hidden
 *     dimension, at block sizes from 4096 (the full hidden size) down to 128;
 *   - quantization error arises both before RS and before AG.
 * Everything else is a reading (the page is silent); each one is stated where
 * it is used.  All arithmetic is binary32 with round-to-nearest-even; this
 * file must be compiled with -ffp-contract=off and without fast-math so that
 * each line below is exactly one IEEE operation.
 *
 * Per block of B values v_0..v_{B-1} (as fp32) at b bits, qmax = 2^b - 1:
 *   mn = min(0, v_i), mx = max(0, v_i)                  range includes zero
 *   d  = mx - mn;  s = (d == 0) ? 1 : d / qmax           fp32 scale
 *   inv = 1 / s                                          per-block reciprocal
 *   z  = clamp(rne(-mn * inv), 0, qmax)                  uint8 zero-point
 *   q_i = clamp(rne(v_i * inv) + z, 0, qmax)             code
 *   xhat_i = (q_i - z) * s                               dequantized value
 * where rne rounds the exact product to the nearest integer, ties to even
 * (one rounding: the product is not first rounded to fp32).
 * INT4 codes are packed two per byte, the even element in the low nibble.
 *
 * Two-step all-reduce over P ranks (rank r holds partial x_r of n elements):
 *   1. every rank quantizes its whole partial (step-1 payload);
 *   2. RS: chunk c (elements [c*n/P, (c+1)*n/P)) is owned by rank c, which
 *      dequantizes that chunk from all P payloads, sums them in fp32 in rank
 *      order 0..P-1 and requantizes the sum (step-2 payload);
 *   3. AG: every rank gathers the P step-2 chunks and dequantizes them to the
 *      fp16/bf16 output; all ranks therefore hold the same output.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define FCO_OK 0
#define FCO_ERR_ARG 1    /* bad sizes, bits, block or rank count      */
#define FCO_ERR_RANGE 2  /* non-finite input, or a block whose range makes
                            the scale or its reciprocal non-finite       */

#define FCO_FP16 0
#define FCO_BF16 1

/* ------------------------------------------------------------------------ */
/* fp16 / bf16 <-> fp32, written from the IEEE-754 binary16 and the bfloat16  */
/* formats.  Widening is exact; narrowing rounds to nearest, ties to even.   */
/* ------------------------------------------------------------------------ */

/* Value of a binary16 bit pattern: sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 is the subnormal range 2^-14 * f/1024. */
float fco_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0x1f)
        v = f ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)f, -24);
    else
        v = ldexp((double)(1024 + f), e - 25);
    return (float)(sign ? -v : v);
}

/* bfloat16 is the upper half of a binary32 pattern. */
float fco_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round |a| (finite, exactly representable in double) to a binary format with
 * `mant` fraction bits and minimum normal exponent `emin`, ties to even.
 * Returns the rounded magnitude as a double (may be above the format's max;
 * the caller decides overflow). */
static double round_to_format(double a, int mant, int emin)
{
    if (a == 0.0)
        return 0.0;
    int ex;
    frexp(a, &ex);              /* a = m * 2^ex, m in [0.5, 1) */
    int e = ex - 1;             /* a in [2^e, 2^(e+1)) */
    if (e < emin)
        e = emin;               /* subnormal spacing */
    double ulp = ldexp(1.0, e - mant);
    double k = a / ulp;         /* exact: power-of-two division */
    double kr = nearbyint(k);   /* ties to even in the default rounding mode */
    return kr * ulp;
}

uint16_t fco_f32_to_f16(float x)
{
    if (isnan(x))
        return 0x7e00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs((double)x);
    double r = round_to_format(a, 10, -14);
    if (r > 65504.0)            /* rounds past the largest finite value */
        return sign | 0x7c00;
    if (r == 0.0)
        return sign;
    if (r < ldexp(1.0, -14))    /* subnormal: fraction counts 2^-24 units */
        return sign | (uint16_t)(r / ldexp(1.0, -24));
    int ex;
    double m = frexp(r, &ex);   /* r = m * 2^ex, m in [0.5,1) */
    int e = ex - 1;
    uint16_t frac = (uint16_t)((m * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)((e + 15) << 10) | frac;
}

uint16_t fco_f32_to_bf16(float x)
{
    if (isnan(x))
        return 0x7fc0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs((double)x);
    double r = round_to_format(a, 7, -126);
    double maxv = ldexp(255.0, 127 - 7);   /* (2 - 2^-7) * 2^127 */
    if (r > maxv)
        return sign | 0x7f80;
    float f = (float)r;                    /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)((u >> 16) & 0x7fff);
}

/* Array forms of the conversions above (used to pin them against library
 * conversions over whole value ranges). */
void fco_widen(const uint16_t* x, int dtype, size_t n, float* out)
{
    for (size_t i = 0; i < n; i++)
        out[i] = dtype == FCO_FP16 ? fco_f16_to_f32(x[i]) : fco_bf16_to_f32(x[i]);
}

void fco_narrow(const float* v, int dtype, size_t n, uint16_t* out)
{
    for (size_t i = 0; i < n; i++)
        out[i] = dtype == FCO_FP16 ? fco_f32_to_f16(v[i]) : fco_f32_to_bf16(v[i]);
}

static float load_elem(const uint16_t* x, size_t i, int dtype)
{
    return dtype == FCO_FP16 ? fco_f16_to_f32(x[i]) : fco_bf16_to_f32(x[i]);
}

static uint16_t store_elem(float v, int dtype)
{
    return dtype == FCO_FP16 ? fco_f32_to_f16(v) : fco_f32_to_bf16(v);
}

/* ------------------------------------------------------------------------ */
/* Per-block asymmetric quantizer (page: TL;DR, activations are quantized   */
/* to low bit widths; Fig. 4, block granularity along hidden).               */
/* ------------------------------------------------------------------------ */

/* Nearest integer, ties to even, of the exact product a*b of two fp32 values.
 * The product of two 24-bit significands has at most 48 bits, so it is exact
 * in double; nearbyint rounds to nearest, ties to even, in the default mode. */
static int rne_product(float a, float b)
{
    double t = (double)a * (double)b;
    return (int)nearbyint(t);
}

static int clamp_int(int v, int lo, int hi)
{
    return v < lo ? lo : (v > hi ? hi : v);
}

/* Scale, reciprocal and zero-point of one block of fp32 values. */
int fco_block_stats(const float* v, int B, int bits, float* s_out, float* inv_out, int* z_out)
{
    const int qmax = (1 << bits) - 1;
    float mn = 0.0f, mx = 0.0f;        /* the range always contains zero */
    for (int i = 0; i < B; i++) {
        if (!isfinite(v[i]))
            return FCO_ERR_RANGE;
        if (v[i] < mn)
            mn = v[i];
        if (v[i] > mx)
            mx = v[i];
    }
    float d = mx - mn;
    float s = (d == 0.0f) ? 1.0f : d / (float)qmax;
    float inv = 1.0f / s;
    if (!isfinite(d) || !isfinite(inv) || s == 0.0f)
        return FCO_ERR_RANGE;
    int z = clamp_int(rne_product(-mn, inv), 0, qmax);
    *s_out = s;
    *inv_out = inv;
    *z_out = z;
    return FCO_OK;
}

/* Code of one value given its block's reciprocal scale and zero-point: round
 * the exact product v*inv first, then add the zero-point as an integer, then
 * clamp. */
int fco_quantize_value(float v, float inv, int z, int bits)
{
    const int qmax = (1 << bits) - 1;
    return clamp_int(rne_product(v, inv) + z, 0, qmax);
}

/* Dequantized value: one fp32 product of the exact integer (q - z) and s. */
float fco_dequantize_value(int q, float s, int z)
{
    float qz = (float)(q - z);
    return qz * s;
}

/* Store / fetch code i of a packed code array (INT4: two per byte, the even
 * element in the low nibble; INT8: one per byte). */
static void put_code(uint8_t* codes, size_t i, int q, int bits)
{
    if (bits == 8) {
        codes[i] = (uint8_t)q;
    } else if (i % 2 == 0) {
        codes[i / 2] = (uint8_t)((codes[i / 2] & 0xf0) | (q & 0x0f));
    } else {
        codes[i / 2] = (uint8_t)((codes[i / 2] & 0x0f) | ((q & 0x0f) << 4));
    }
}

static int get_code(const uint8_t* codes, size_t i, int bits)
{
    if (bits == 8)
        return codes[i];
    return (i % 2 == 0) ? (codes[i / 2] & 0x0f) : (codes[i / 2] >> 4);
}

static int check_shape(size_t n, int bits, int block)
{
    if (bits != 4 && bits != 8)
        return FCO_ERR_ARG;
    if (block < 2 || (block % 2) != 0)
        return FCO_ERR_ARG;
    if (n % (size_t)block != 0)
        return FCO_ERR_ARG;
    return FCO_OK;
}

/* Quantize a block of fp32 values into the payload at block index k. */
static int quantize_block(const float* v, int B, int bits, size_t k,
                          uint8_t* codes, float* scales, uint8_t* zps)
{
    float s, inv;
    int z;
    int st = fco_block_stats(v, B, bits, &s, &inv, &z);
    if (st != FCO_OK)
        return st;
    for (int i = 0; i < B; i++)
        put_code(codes, k * (size_t)B + (size_t)i, fco_quantize_value(v[i], inv, z, bits), bits);
    scales[k] = s;
    zps[k] = (uint8_t)z;
    return FCO_OK;
}

/* Step 1 on one rank: quantize n fp16/bf16 values block by block. */
int fco_quantize(const uint16_t* x, int dtype, size_t n, int bits, int block,
                 uint8_t* codes, float* scales, uint8_t* zps)
{
    int st = check_shape(n, bits, block);
    if (st != FCO_OK || (dtype != FCO_FP16 && dtype != FCO_BF16))
        return FCO_ERR_ARG;
    float* v = (float*)malloc(sizeof(float) * (size_t)block);
    if (!v)
        return FCO_ERR_ARG;
    for (size_t k = 0; k < n / (size_t)block; k++) {
        for (int i = 0; i < block; i++)
            v[i] = load_elem(x, k * (size_t)block + (size_t)i, dtype);
        st = quantize_block(v, block, bits, k, codes, scales, zps);
        if (st != FCO_OK)
            break;
    }
    free(v);
    return st;
}

/* The same quantizer on fp32 values (the form the reduce-scatter step applies
 * to its fp32 sums). */
int fco_quantize_f32(const float* v, size_t n, int bits, int block,
                     uint8_t* codes, float* scales, uint8_t* zps)
{
    int st = check_shape(n, bits, block);
    if (st != FCO_OK)
        return st;
    for (size_t k = 0; k < n / (size_t)block && st == FCO_OK; k++)
        st = quantize_block(v + k * (size_t)block, block, bits, k, codes, scales, zps);
    return st;
}

/* Dequantize a whole payload to fp32 (xhat), block by block. */
int fco_dequantize(const uint8_t* codes, const float* scales, const uint8_t* zps,
                   size_t n, int bits, int block, float* out)
{
    int st = check_shape(n, bits, block);
    if (st != FCO_OK)
        return st;
    for (size_t i = 0; i < n; i++) {
        size_t k = i / (size_t)block;
        out[i] = fco_dequantize_value(get_code(codes, i, bits), scales[k], zps[k]);
    }
    return FCO_OK;
}

/* Step 2, reduce-scatter: for each chunk c (owned by rank c), dequantize the
 * chunk from all P step-1 payloads, sum in fp32 in rank order 0..P-1 (the sum
 * starts from rank 0's value; no fused multiply-add), and requantize the sum
 * block by block into the step-2 payload.  The owner's own contribution goes
 * through quantization too.  Chunks are block-aligned: n % (P*block) == 0. */
int fco_rs_dequant_sum_requant(const uint8_t* const* codes, const float* const* scales,
                               const uint8_t* const* zps, int P, size_t n, int bits, int block,
                               uint8_t* codes2, float* scales2, uint8_t* zps2)
{
    int st = check_shape(n, bits, block);
    if (st != FCO_OK || P < 1 || n % ((size_t)P * (size_t)block) != 0)
        return FCO_ERR_ARG;
    const size_t chunk = n / (size_t)P;
    float* acc = (float*)malloc(sizeof(float) * (size_t)block);
    if (!acc)
        return FCO_ERR_ARG;
    for (int c = 0; c < P && st == FCO_OK; c++) {
        for (size_t b0 = (size_t)c * chunk; b0 < (size_t)(c + 1) * chunk; b0 += (size_t)block) {
            size_t k = b0 / (size_t)block;
            for (int i = 0; i < block; i++) {
                size_t e = b0 + (size_t)i;
                float a = fco_dequantize_value(get_code(codes[0], e, bits), scales[0][k], zps[0][k]);
                for (int r = 1; r < P; r++) {
                    float xr = fco_dequantize_value(get_code(codes[r], e, bits), scales[r][k], zps[r][k]);
                    a = a + xr;
                }
                acc[i] = a;
            }
            st = quantize_block(acc, block, bits, k, codes2, scales2, zps2);
            if (st != FCO_OK)
                break;
        }
    }
    free(acc);
    return st;
}

/* Step 3, all-gather: every chunk of the step-2 payload is dequantized and
 * rounded (to nearest, ties to even) to the fp16/bf16 output. */
int fco_ag_dequant(const uint8_t* codes2, const float* scales2, const uint8_t* zps2,
                   size_t n, int bits, int block, int out_dtype, uint16_t* y)
{
    int st = check_shape(n, bits, block);
    if (st != FCO_OK || (out_dtype != FCO_FP16 && out_dtype != FCO_BF16))
        return FCO_ERR_ARG;
    for (size_t i = 0; i < n; i++) {
        size_t k = i / (size_t)block;
        float v = fco_dequantize_value(get_code(codes2, i, bits), scales2[k], zps2[k]);
        y[i] = store_elem(v, out_dtype);
    }
    return FCO_OK;
}

/* The whole two-step all-reduce: step 1 on every rank, RS, AG.  The step-1
 * payloads (P arrays each of codes/scales/zps) and the step-2 payload are
 * outputs here as well; the caller provides all of them. */
int fco_allreduce(const uint16_t* const* x, int P, int dtype, size_t n, int bits, int block,
                  uint8_t* const* codes1, float* const* scales1, uint8_t* const* zps1,
                  uint8_t* codes2, float* scales2, uint8_t* zps2, uint16_t* y)
{
    int st = check_shape(n, bits, block);
    if (st != FCO_OK || P < 1 || n % ((size_t)P * (size_t)block) != 0)
        return FCO_ERR_ARG;
    for (int r = 0; r < P; r++) {
        st = fco_quantize(x[r], dtype, n, bits, block, codes1[r], scales1[r], zps1[r]);
        if (st != FCO_OK)
            return st;
    }
    st = fco_rs_dequant_sum_requant((const uint8_t* const*)codes1, (const float* const*)scales1,
                                    (const uint8_t* const*)zps1, P, n, bits, block,
                                    codes2, scales2, zps2);
    if (st != FCO_OK)
        return st;
    return fco_ag_dequant(codes2, scales2, zps2, n, bits, block, dtype, y);
}

/* ------------------------------------------------------------------------ */
/* Per-step precision (page: Fig. 5 right compares the quantization error   */
/* of the reduce-scatter step with that of the all-gather step).  bits_rs    */
/* and bits_ag are each                                                      */
/* 4, 8 or 16; 16 means that step sends the 16-bit values unquantized:        */
/*   bits_rs == 16: the RS sums the exactly widened inputs x_r;              */
/*   bits_ag == 16: the AG sends the fp32 sum rounded to fp16/bf16, so the    */
/*                  output is that rounding.                                 */
/* With bits_rs == bits_ag == b this is fco_allreduce.  Payload outputs of a  */
/* step that is not quantized are not written (they may be NULL).            */
/* ------------------------------------------------------------------------ */
int fco_allreduce_ex(const uint16_t* const* x, int P, int dtype, size_t n, int bits_rs, int bits_ag,
                     int block, uint8_t* const* codes1, float* const* scales1, uint8_t* const* zps1,
                     uint8_t* codes2, float* scales2, uint8_t* zps2, uint16_t* y)
{
    int bq = bits_rs != 16 ? bits_rs : (bits_ag != 16 ? bits_ag : 8);
    int st = check_shape(n, bq, block);
    if (st != FCO_OK || P < 1 || n % ((size_t)P * (size_t)block) != 0 ||
        (bits_rs != 4 && bits_rs != 8 && bits_rs != 16) || (bits_ag != 4 && bits_ag != 8 && bits_ag != 16) ||
        (dtype != FCO_FP16 && dtype != FCO_BF16))
        return FCO_ERR_ARG;
    /* step 1: every rank's contribution as the RS receives it */
    float* contrib = (float*)malloc(sizeof(float) * n * (size_t)P);
    float* acc = (float*)malloc(sizeof(float) * (size_t)block);
    if (!contrib || !acc) {
        free(contrib);
        free(acc);
        return FCO_ERR_ARG;
    }
    for (int r = 0; r < P && st == FCO_OK; r++) {
        float* c = contrib + (size_t)r * n;
        if (bits_rs == 16) {
            for (size_t i = 0; i < n; i++)
                c[i] = load_elem(x[r], i, dtype);
        } else {
            st = fco_quantize(x[r], dtype, n, bits_rs, block, codes1[r], scales1[r], zps1[r]);
            if (st == FCO_OK)
                st = fco_dequantize(codes1[r], scales1[r], zps1[r], n, bits_rs, block, c);
        }
    }
    /* RS per owned chunk, then AG of every chunk */
    const size_t chunk = n / (size_t)P;
    for (int cidx = 0; cidx < P && st == FCO_OK; cidx++) {
        for (size_t b0 = (size_t)cidx * chunk; b0 < (size_t)(cidx + 1) * chunk && st == FCO_OK;
             b0 += (size_t)block) {
            size_t k = b0 / (size_t)block;
            for (int i = 0; i < block; i++) {
                float a = contrib[b0 + (size_t)i];
                for (int r = 1; r < P; r++)
                    a = a + contrib[(size_t)r * n + b0 + (size_t)i];
                acc[i] = a;
            }
            if (bits_ag == 16) {
                for (int i = 0; i < block; i++)
                    y[b0 + (size_t)i] = store_elem(acc[i], dtype);
            } else {
                st = quantize_block(acc, block, bits_ag, k, codes2, scales2, zps2);
                for (int i = 0; i < block && st == FCO_OK; i++) {
                    size_t e = b0 + (size_t)i;
                    float v = fco_dequantize_value(get_code(codes2, e, bits_ag), scales2[k], zps2[k]);
                    y[e] = store_elem(v, dtype);
                }
            }
        }
    }
    free(contrib);
    free(acc);
    return st;
}

