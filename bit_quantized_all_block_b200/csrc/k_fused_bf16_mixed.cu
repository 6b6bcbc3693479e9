// Instantiations of the fused all-reduce kernel with per-step widths (reduce-scatter
// bits, all-gather bits; 16 = that step unquantized) for __nv_bfloat16, P = 2, 4, 8.
#include "fc_launch_impl.cuh"

namespace fc {
template cudaError_t launch_fused<__nv_bfloat16, 8, 4, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 4, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 4, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 8, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 8, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 8, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 8, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 8, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 8, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 4, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 4, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 4, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 16, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 16, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 16, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 16, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 16, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 16, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 16, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 16, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 16, 16, 8>(const FusedArgs&, cudaStream_t);
}  // namespace fc
