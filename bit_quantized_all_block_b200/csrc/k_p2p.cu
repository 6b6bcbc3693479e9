// Instantiations of the one-kernel P-GPU all-reduce (fc_p2p.cuh): fp16/bf16,
// INT8/INT4, P = 2, 4, 8, per rank and emulated (all ranks in one launch).
#include "fc_p2p.cuh"

namespace fc {
#define FC_P2P(T, B, P)                                                                 \
    template cudaError_t launch_p2p<T, B, P, false>(const P2PArgs&, int, cudaStream_t); \
    template cudaError_t launch_p2p<T, B, P, true>(const P2PArgs&, int, cudaStream_t);  \
    template cudaError_t p2p_max_ctas<T, B, P, false>(int*);                            \
    template cudaError_t p2p_max_ctas<T, B, P, true>(int*);
FC_P2P(__half, 8, 2) FC_P2P(__half, 8, 4) FC_P2P(__half, 8, 8)
FC_P2P(__half, 4, 2) FC_P2P(__half, 4, 4) FC_P2P(__half, 4, 8)
FC_P2P(__nv_bfloat16, 8, 2) FC_P2P(__nv_bfloat16, 8, 4) FC_P2P(__nv_bfloat16, 8, 8)
FC_P2P(__nv_bfloat16, 4, 2) FC_P2P(__nv_bfloat16, 4, 4) FC_P2P(__nv_bfloat16, 4, 8)
#undef FC_P2P
}  // namespace fc
