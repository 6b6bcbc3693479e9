// The packed fp32 pair operations of the library, and its dequantize-and-
// accumulate step built from them, against the scalar binary32 operations they
// stand for (test infrastructure: built and run by tests/test_gpu_packed.py on
// a GPU).  Inputs come from a counter-based hash, so nothing but a mismatch
// counter lives in device memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../bit_quantized_all_block_b200/csrc/fc_device.cuh"

__device__ __forceinline__ uint32_t mix(uint64_t x)
{
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return (uint32_t)(x ^ (x >> 31));
}

// A finite float from random bits (exponent field 0xFF replaced).
__device__ __forceinline__ float finite(uint32_t u)
{
    if ((u & 0x7F800000u) == 0x7F800000u)
        u &= 0xBFFFFFFFu;
    return __uint_as_float(u);
}

__device__ __forceinline__ bool same(float a, float b) { return __float_as_uint(a) == __float_as_uint(b); }

// WHICH 0: add2 / mul2 / fma2 lane by lane on arbitrary finite operands.
// WHICH 1: the rank-order accumulation step acc + (sh - mz) * s in both forms
//          the kernels use (a packed subtract, then prod2 and a packed add, or
//          mul2 and scalar adds), on shifted codes
//          sh = 1.5*2^23 + q, mz = 1.5*2^23 + z, q, z in [0, 255], a random
//          scale and a random running sum -- two roundings, as the scalar chain.
template <int WHICH>
__global__ void k_check(uint64_t n, uint32_t seed, unsigned long long* bad)
{
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t base = ((uint64_t)seed << 40) ^ (i * 8);
        const uint32_t r0 = mix(base), r1 = mix(base + 1), r2 = mix(base + 2), r3 = mix(base + 3);  // r2: WHICH 0 only
        const uint32_t r4 = mix(base + 4), r5 = mix(base + 5);
        int wrong = 0;
        if (WHICH == 0) {
            const float2 a = make_float2(finite(r0), finite(r1)), b = make_float2(finite(r2), finite(r3));
            const float2 c = make_float2(finite(r4), finite(r5));
            const float2 s = fc::add2(a, b), m = fc::mul2(a, b), f = fc::fma2(a, b, c), p = fc::prod2(a, b);
            // prod2 equals the product except for the sign of an exact zero product
            // (+0 instead of -0), which the kernels never form: their scale is
            // positive and their integer factor is never -0
            const bool px = a.x != 0.0f && b.x != 0.0f, py = a.y != 0.0f && b.y != 0.0f;
            wrong = !same(s.x, __fadd_rn(a.x, b.x)) || !same(s.y, __fadd_rn(a.y, b.y)) ||
                    (px && !same(p.x, __fmul_rn(a.x, b.x))) || (py && !same(p.y, __fmul_rn(a.y, b.y))) ||
                    !same(m.x, __fmul_rn(a.x, b.x)) || !same(m.y, __fmul_rn(a.y, b.y)) ||
                    !same(f.x, __fmaf_rn(a.x, b.x, c.x)) || !same(f.y, __fmaf_rn(a.y, b.y, c.y));
        } else {
            const float sh0 = fc::FC_MAGIC + (float)(r0 & 255u), sh1 = fc::FC_MAGIC + (float)((r0 >> 8) & 255u);
            const float mz = fc::FC_MAGIC + (float)((r0 >> 16) & 255u);
            const float s = __uint_as_float(0x30000000u + (r1 & 0x0FFFFFFFu));    // about 2^-31 .. 2^-1
            float acc[2] = {__uint_as_float(0x30000000u + (r3 & 0x1FFFFFFFu)),
                            -__uint_as_float(0x30000000u + (r4 & 0x1FFFFFFFu))};
            const float want0 = __fadd_rn(acc[0], __fmul_rn(__fsub_rn(sh0, mz), s));
            const float want1 = __fadd_rn(acc[1], __fmul_rn(__fsub_rn(sh1, mz), s));
            // the two forms the kernels use: prod2 then a packed add; mul2 then scalar adds
            float acc2[2] = {acc[0], acc[1]};
            const float2 t = fc::add2(make_float2(sh0, sh1), fc::dup2(-mz));
            fc::st2(acc, 0, fc::add2(fc::ld2(acc, 0), fc::prod2(t, fc::dup2(s))));
            fc::acc_add(acc2, 0, fc::mul2(t, fc::dup2(s)));
            wrong = !same(acc[0], want0) || !same(acc[1], want1) || !same(acc2[0], want0) || !same(acc2[1], want1);
        }
        if (wrong)
            atomicAdd(bad, 1ull);
    }
}

extern "C" int fc_check_packed(int which, unsigned long long n, unsigned int seed, unsigned long long* bad_out)
{
    unsigned long long* bad = nullptr;
    if (cudaMalloc(&bad, sizeof(*bad)) != cudaSuccess)
        return 1;
    cudaMemset(bad, 0, sizeof(*bad));
    if (which == 0)
        k_check<0><<<148 * 8, 256>>>(n, seed, bad);
    else
        k_check<1><<<148 * 8, 256>>>(n, seed, bad);
    cudaError_t e = cudaMemcpy(bad_out, bad, sizeof(*bad), cudaMemcpyDeviceToHost);
    cudaFree(bad);
    return e == cudaSuccess ? 0 : 2;
}
