// Instantiations of the fused all-reduce kernel for blocks whose thread group is
// narrower than P lanes (the scale of every rank computed by every lane): __nv_bfloat16,
// quantized reduce-scatter, P = 3..8 for equal widths, P = 4, 8 for the others.
#include "fc_launch_impl.cuh"

namespace fc {
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 3, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 4, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 5, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 6, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 7, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 8, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 3, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 4, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 5, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 6, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 7, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 8, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 4, 4, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 4, 8, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 8, 4, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 8, 8, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 16, 4, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 16, 8, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 16, 4, false, false, false>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 16, 8, false, false, false>(const FusedArgs&, cudaStream_t);
}  // namespace fc
