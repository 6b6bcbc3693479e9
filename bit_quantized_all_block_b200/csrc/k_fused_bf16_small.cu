// Instantiations of the fused all-reduce kernel in its latency shape (decode-sized
// messages): __nv_bfloat16, equal widths INT8 / INT4, P = 2, 4, 8.
#include "fc_launch_impl.cuh"

namespace fc {
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 2, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 4, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 8, 8, 8, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 2, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 4, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__nv_bfloat16, 4, 4, 8, true>(const FusedArgs&, cudaStream_t);
}  // namespace fc
