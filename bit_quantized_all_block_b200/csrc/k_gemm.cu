// Launchers and instantiations of the GEMM with the fused step-1 quantizer
// (fp16/bf16 operands, INT8/INT4 codes, quantization blocks of 32/64/128/256).
#include <cuda_runtime.h>

#include <map>
#include <mutex>

#include "fc_gemm.cuh"

namespace fc {

template <class T, int BITS, int NB>
cudaError_t launch_gemm_quant(const CUtensorMap& ta, const CUtensorMap& tb, const GemmQuantArgs& a,
                              cudaStream_t st)
{
    static std::mutex mu;
    static std::map<int, int> sms_of;   // device -> SM count, with the smem attribute set
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    int sms = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = sms_of.find(dev);
        if (it == sms_of.end()) {
            e = cudaFuncSetAttribute(k_gemm_quant<T, BITS, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     GQ_SMEM_BYTES);
            if (e != cudaSuccess)
                return e;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess)
                return e;
            sms_of[dev] = sms;
        } else {
            sms = it->second;
        }
    }
    const int tiles = a.tiles_m * a.tiles_n;
    const int grid = tiles < sms ? tiles : sms;
    k_gemm_quant<T, BITS, NB><<<grid, GQ_THREADS, GQ_SMEM_BYTES, st>>>(ta, tb, a);
    return cudaGetLastError();
}

template <class T, int BITS, int NB>
cudaError_t launch_gemm_quant_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmQuantArgs& a,
                                   cudaStream_t st)
{
    static std::mutex mu;
    static std::map<int, int> sms_of;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    int sms = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = sms_of.find(dev);
        if (it == sms_of.end()) {
            e = cudaFuncSetAttribute(k_gemm_quant_pair<T, BITS, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     G2_SMEM_BYTES);
            if (e != cudaSuccess)
                return e;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess)
                return e;
            sms_of[dev] = sms;
        } else {
            sms = it->second;
        }
    }
    const int pairs_needed = (a.tiles_m / 2) * a.tiles_n;
    const int pairs = pairs_needed < sms / 2 ? pairs_needed : sms / 2;
    k_gemm_quant_pair<T, BITS, NB><<<2 * pairs, GQ_THREADS, G2_SMEM_BYTES, st>>>(ta, tb, a);
    return cudaGetLastError();
}

#define FC_GQ(T)                                                                                  \
    template cudaError_t launch_gemm_quant<T, 8, 32>(const CUtensorMap&, const CUtensorMap&,      \
                                                     const GemmQuantArgs&, cudaStream_t);         \
    template cudaError_t launch_gemm_quant<T, 8, 64>(const CUtensorMap&, const CUtensorMap&,      \
                                                     const GemmQuantArgs&, cudaStream_t);         \
    template cudaError_t launch_gemm_quant<T, 8, 128>(const CUtensorMap&, const CUtensorMap&,     \
                                                      const GemmQuantArgs&, cudaStream_t);        \
    template cudaError_t launch_gemm_quant<T, 4, 32>(const CUtensorMap&, const CUtensorMap&,      \
                                                     const GemmQuantArgs&, cudaStream_t);         \
    template cudaError_t launch_gemm_quant<T, 4, 64>(const CUtensorMap&, const CUtensorMap&,      \
                                                     const GemmQuantArgs&, cudaStream_t);         \
    template cudaError_t launch_gemm_quant<T, 4, 128>(const CUtensorMap&, const CUtensorMap&,     \
                                                      const GemmQuantArgs&, cudaStream_t);        \
    template cudaError_t launch_gemm_quant<T, 8, 256>(const CUtensorMap&, const CUtensorMap&,     \
                                                      const GemmQuantArgs&, cudaStream_t);        \
    template cudaError_t launch_gemm_quant<T, 4, 256>(const CUtensorMap&, const CUtensorMap&,     \
                                                      const GemmQuantArgs&, cudaStream_t);
FC_GQ(__half)
FC_GQ(__nv_bfloat16)
#undef FC_GQ

#define FC_GQ2(T, B, NB)                                                                           \
    template cudaError_t launch_gemm_quant_pair<T, B, NB>(const CUtensorMap&, const CUtensorMap&,  \
                                                          const GemmQuantArgs&, cudaStream_t);
FC_GQ2(__half, 8, 32) FC_GQ2(__half, 8, 64) FC_GQ2(__half, 8, 128)
FC_GQ2(__half, 4, 32) FC_GQ2(__half, 4, 64) FC_GQ2(__half, 4, 128)
FC_GQ2(__nv_bfloat16, 8, 32) FC_GQ2(__nv_bfloat16, 8, 64) FC_GQ2(__nv_bfloat16, 8, 128)
FC_GQ2(__nv_bfloat16, 4, 32) FC_GQ2(__nv_bfloat16, 4, 64) FC_GQ2(__nv_bfloat16, 4, 128)
FC_GQ2(__half, 8, 256) FC_GQ2(__half, 4, 256) FC_GQ2(__nv_bfloat16, 8, 256) FC_GQ2(__nv_bfloat16, 4, 256)
#undef FC_GQ2

}  // namespace fc
