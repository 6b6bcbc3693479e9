// Instantiations of the fused all-reduce kernel: __nv_bfloat16, INT4 in both steps, P = 1..8, with
// 16-byte and with 32-byte global accesses.
#include "fc_launch_impl.cuh"

namespace fc {
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 1>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 3>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 5>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 6>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 7>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 1, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 2, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 3, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 4, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 5, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 6, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 7, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 8, false, true>(const FusedArgs&, cudaStream_t);
}  // namespace fc
