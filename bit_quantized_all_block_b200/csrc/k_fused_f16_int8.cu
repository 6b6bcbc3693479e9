// Instantiations of the fused all-reduce kernel: __half, INT8 in both steps, P = 1..8, with
// 16-byte and with 32-byte global accesses.
#include "fc_launch_impl.cuh"

namespace fc {
template cudaError_t launch_fused<__half, 8, 8, 1>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 2>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 3>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 4>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 5>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 6>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 7>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 8>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 1, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 2, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 3, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 4, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 5, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 6, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 7, false, true>(const FusedArgs&, cudaStream_t);
template cudaError_t launch_fused<__half, 8, 8, 8, false, true>(const FusedArgs&, cudaStream_t);
}  // namespace fc
