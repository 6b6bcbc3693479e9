// The GEMM pipeline's bounded wait gives up instead of hanging (test
// infrastructure: built and run by tests/test_gpu_wait_timeout.py).  One
// thread waits on an mbarrier that nothing ever arrives on; the wait must
// return false after the library's time limit, raise the abort flag, and
// leave the context usable.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../bit_quantized_all_block_b200/csrc/fc_gemm.cuh"

__global__ void k_wait_never(unsigned long long* out)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        fc::mbar_init(&bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = fc::global_ns();
        const bool ok = fc::wait_bounded(&bar, 0, &abort_flag);
        out[0] = ok ? 1ull : 0ull;
        out[1] = (unsigned long long)abort_flag;
        out[2] = fc::global_ns() - t0;
    }
}

__global__ void k_still_alive(unsigned long long* out) { out[3] = 42; }

extern "C" int fc_check_wait_timeout(unsigned long long* host_out)
{
    unsigned long long* d = nullptr;
    if (cudaMalloc(&d, 4 * sizeof(unsigned long long)) != cudaSuccess)
        return 1;
    cudaMemset(d, 0xff, 4 * sizeof(unsigned long long));
    k_wait_never<<<1, 32>>>(d);
    cudaError_t e1 = cudaDeviceSynchronize();
    k_still_alive<<<1, 1>>>(d);
    cudaError_t e2 = cudaDeviceSynchronize();
    cudaMemcpy(host_out, d, 4 * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
    cudaFree(d);
    return (e1 == cudaSuccess && e2 == cudaSuccess) ? 0 : 2;
}
