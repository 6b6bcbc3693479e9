// Instantiations of the staged kernels: step-1 quantize, reduce-scatter
// (P = 1..8) and all-gather dequantize, for fp16/bf16 and INT8/INT4.
#include "fc_launch_impl.cuh"

namespace fc {
template cudaError_t launch_quantize<__half, 8>(const QuantArgs&, cudaStream_t);
template cudaError_t launch_quantize<__half, 4>(const QuantArgs&, cudaStream_t);
template cudaError_t launch_quantize<__nv_bfloat16, 8>(const QuantArgs&, cudaStream_t);
template cudaError_t launch_quantize<__nv_bfloat16, 4>(const QuantArgs&, cudaStream_t);
template cudaError_t launch_ag<__half, 8>(const AgArgs&, cudaStream_t);
template cudaError_t launch_ag<__half, 4>(const AgArgs&, cudaStream_t);
template cudaError_t launch_ag<__nv_bfloat16, 8>(const AgArgs&, cudaStream_t);
template cudaError_t launch_ag<__nv_bfloat16, 4>(const AgArgs&, cudaStream_t);
template cudaError_t launch_ag<__half, 8, true>(const AgArgs&, cudaStream_t);
template cudaError_t launch_ag<__half, 4, true>(const AgArgs&, cudaStream_t);
template cudaError_t launch_ag<__nv_bfloat16, 8, true>(const AgArgs&, cudaStream_t);
template cudaError_t launch_ag<__nv_bfloat16, 4, true>(const AgArgs&, cudaStream_t);
#define FC_RS(BITS, P) template cudaError_t launch_rs<BITS, P>(const RsArgs&, cudaStream_t);
FC_RS(8, 1) FC_RS(8, 2) FC_RS(8, 3) FC_RS(8, 4) FC_RS(8, 5) FC_RS(8, 6) FC_RS(8, 7) FC_RS(8, 8)
FC_RS(4, 1) FC_RS(4, 2) FC_RS(4, 3) FC_RS(4, 4) FC_RS(4, 5) FC_RS(4, 6) FC_RS(4, 7) FC_RS(4, 8)
#undef FC_RS
}  // namespace fc
