/*
 * A C caller of the library's C ABI (include/fc.h) with no Python and no
 * torch: device memory from the CUDA driver API, the fused all-reduce and the
 * three staged steps on the legacy default stream, results compared bit for
 * bit with the CPU oracle's C definition (test infrastructure: built with gcc
 * and run by tests/test_gpu_abi_c.py on a GPU).
 *
 *   abi_c_check P dtype bits block n seed      (dtype 0 = fp16, 1 = bf16)
 *
 * Exit status 0 when every output and payload byte agrees, 1 on a mismatch,
 * 2 on a setup or API error.
 */
#include <cuda.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "../../include/fc.h"

/* The oracle's entry point (oracle/fco.c, linked from libfco.so). */
int fco_allreduce(const uint16_t* const* x, int P, int dtype, size_t n, int bits, int block,
                  uint8_t* const* codes1, float* const* scales1, uint8_t* const* zps1, uint8_t* codes2,
                  float* scales2, uint8_t* zps2, uint16_t* y);

#define CK(call)                                                                   \
    do {                                                                           \
        CUresult r_ = (call);                                                      \
        if (r_ != CUDA_SUCCESS) {                                                  \
            fprintf(stderr, "%s failed: %d\n", #call, (int)r_);                    \
            exit(2);                                                               \
        }                                                                          \
    } while (0)
#define FC(call)                                                                   \
    do {                                                                           \
        fc_status s_ = (call);                                                     \
        if (s_ != FC_OK) {                                                         \
            fprintf(stderr, "%s: %s\n", #call, fc_status_string(s_));              \
            exit(2);                                                               \
        }                                                                          \
    } while (0)

static uint64_t state;
static uint32_t next32(void)
{
    state = state * 6364136223846793005ull + 1442695040888963407ull;
    return (uint32_t)(state >> 32);
}

/* A finite fp16 / bf16 bit pattern of moderate magnitude (2^-6 .. 2^6). */
static uint16_t random_value(int dtype)
{
    uint32_t r = next32();
    uint16_t sign = (uint16_t)((r >> 31) << 15);
    if (dtype == FC_FP16) {
        uint16_t e = (uint16_t)(9 + (r >> 10) % 13); /* biased exponent 9..21 */
        return (uint16_t)(sign | (e << 10) | (r & 0x3FF));
    }
    uint16_t e = (uint16_t)(121 + (r >> 7) % 13);    /* biased exponent 121..133 */
    return (uint16_t)(sign | (e << 7) | (r & 0x7F));
}

static CUdeviceptr dalloc(size_t bytes)
{
    CUdeviceptr p = 0;
    CK(cuMemAlloc(&p, bytes ? bytes : 16));
    return p;
}

static int same(const void* a, const void* b, size_t bytes, const char* what)
{
    if (memcmp(a, b, bytes) != 0) {
        const uint8_t *x = (const uint8_t*)a, *y = (const uint8_t*)b;
        size_t i = 0;
        while (x[i] == y[i])
            i++;
        fprintf(stderr, "%s differs at byte %zu\n", what, i);
        return 0;
    }
    return 1;
}

int main(int argc, char** argv)
{
    if (argc != 7) {
        fprintf(stderr, "usage: %s P dtype bits block n seed\n", argv[0]);
        return 2;
    }
    const int P = atoi(argv[1]), dtype = atoi(argv[2]), bits = atoi(argv[3]), block = atoi(argv[4]);
    const size_t n = (size_t)strtoull(argv[5], NULL, 10);
    state = (uint64_t)strtoull(argv[6], NULL, 10);
    if (P < 1 || P > 8)
        return 2;

    CUdevice dev;
    CUcontext ctx;
    CK(cuInit(0));
    CK(cuDeviceGet(&dev, 0));
    CK(cuDevicePrimaryCtxRetain(&ctx, dev));
    CK(cuCtxSetCurrent(ctx));

    size_t cb = 0, nb = 0;
    FC(fc_payload_sizes(n, bits, block, &cb, &nb));

    /* host inputs and the oracle's results */
    uint16_t* hx[8];
    uint8_t *oc1[8], *oz1[8];
    float* os1[8];
    for (int r = 0; r < P; r++) {
        hx[r] = (uint16_t*)malloc(n * 2);
        for (size_t i = 0; i < n; i++)
            hx[r][i] = random_value(dtype);
        oc1[r] = (uint8_t*)malloc(cb + 1);
        os1[r] = (float*)malloc(nb * 4 + 4);
        oz1[r] = (uint8_t*)malloc(nb + 1);
    }
    uint8_t* oc2 = (uint8_t*)malloc(cb + 1);
    float* os2 = (float*)malloc(nb * 4 + 4);
    uint8_t* oz2 = (uint8_t*)malloc(nb + 1);
    uint16_t* oy = (uint16_t*)malloc(n * 2 + 2);
    if (fco_allreduce((const uint16_t* const*)hx, P, dtype, n, bits, block, oc1, os1, oz1, oc2, os2, oz2, oy) != 0) {
        fprintf(stderr, "oracle rejected the inputs\n");
        return 2;
    }

    /* device buffers: inputs, the fused call's output and payloads, the staged path's */
    void* dx[8];
    fc_qbuf f1[8], s1[8], f2, s2;
    for (int r = 0; r < P; r++) {
        CUdeviceptr p = dalloc(n * 2);
        CK(cuMemcpyHtoD(p, hx[r], n * 2));
        dx[r] = (void*)(uintptr_t)p;
        f1[r].codes = (uint8_t*)(uintptr_t)dalloc(cb);
        f1[r].scales = (float*)(uintptr_t)dalloc(nb * 4);
        f1[r].zps = (uint8_t*)(uintptr_t)dalloc(nb);
        s1[r].codes = (uint8_t*)(uintptr_t)dalloc(cb);
        s1[r].scales = (float*)(uintptr_t)dalloc(nb * 4);
        s1[r].zps = (uint8_t*)(uintptr_t)dalloc(nb);
    }
    f2.codes = (uint8_t*)(uintptr_t)dalloc(cb);
    f2.scales = (float*)(uintptr_t)dalloc(nb * 4);
    f2.zps = (uint8_t*)(uintptr_t)dalloc(nb);
    s2.codes = (uint8_t*)(uintptr_t)dalloc(cb);
    s2.scales = (float*)(uintptr_t)dalloc(nb * 4);
    s2.zps = (uint8_t*)(uintptr_t)dalloc(nb);
    CUdeviceptr y1 = dalloc(n * 2), y2 = dalloc(n * 2);

    /* argument validation happens on the host, before anything is launched */
    if (fc_quantized_allreduce((const void* const*)dx, P, (fc_dtype)dtype, n, 3, block, (void*)(uintptr_t)y1, NULL,
                               NULL, NULL) != FC_ERR_INVALID_ARG) {
        fprintf(stderr, "bits = 3 was not rejected\n");
        return 1;
    }

    FC(fc_quantized_allreduce((const void* const*)dx, P, (fc_dtype)dtype, n, bits, block, (void*)(uintptr_t)y1, f1,
                              &f2, NULL));
    for (int r = 0; r < P; r++)
        FC(fc_quantize(dx[r], (fc_dtype)dtype, n, bits, block, &s1[r], NULL));
    FC(fc_rs_dequant_sum_requant(s1, P, n, bits, block, &s2, NULL));
    FC(fc_ag_dequant(&s2, n, bits, block, (fc_dtype)dtype, (void*)(uintptr_t)y2, NULL));
    CK(cuCtxSynchronize());

    int ok = 1;
    uint8_t* hb = (uint8_t*)malloc(n * 2 + nb * 4 + cb + 16);
    CK(cuMemcpyDtoH(hb, y1, n * 2));
    ok &= same(hb, oy, n * 2, "fused output");
    CK(cuMemcpyDtoH(hb, y2, n * 2));
    ok &= same(hb, oy, n * 2, "staged output");
    for (int r = 0; r < P; r++) {
        const fc_qbuf* q[2] = {&f1[r], &s1[r]};
        for (int v = 0; v < 2; v++) {
            CK(cuMemcpyDtoH(hb, (CUdeviceptr)(uintptr_t)q[v]->codes, cb));
            ok &= same(hb, oc1[r], cb, "step-1 codes");
            CK(cuMemcpyDtoH(hb, (CUdeviceptr)(uintptr_t)q[v]->scales, nb * 4));
            ok &= same(hb, os1[r], nb * 4, "step-1 scales");
            CK(cuMemcpyDtoH(hb, (CUdeviceptr)(uintptr_t)q[v]->zps, nb));
            ok &= same(hb, oz1[r], nb, "step-1 zero-points");
        }
    }
    const fc_qbuf* q2[2] = {&f2, &s2};
    for (int v = 0; v < 2; v++) {
        CK(cuMemcpyDtoH(hb, (CUdeviceptr)(uintptr_t)q2[v]->codes, cb));
        ok &= same(hb, oc2, cb, "step-2 codes");
        CK(cuMemcpyDtoH(hb, (CUdeviceptr)(uintptr_t)q2[v]->scales, nb * 4));
        ok &= same(hb, os2, nb * 4, "step-2 scales");
        CK(cuMemcpyDtoH(hb, (CUdeviceptr)(uintptr_t)q2[v]->zps, nb));
        ok &= same(hb, oz2, nb, "step-2 zero-points");
    }
    printf("%s: P=%d dtype=%d bits=%d block=%d n=%zu\n", ok ? "ok" : "MISMATCH", P, dtype, bits, block, n);
    CK(cuDevicePrimaryCtxRelease(dev));
    return ok ? 0 : 1;
}
