// fc_p2p_args.cuh -- arguments and launchers of the one-kernel P-GPU all-reduce
// (kernel in fc_p2p.cuh; host entry points in fc_api.cu).
#pragma once

#include "fc_kernels.cuh"

namespace fc {

constexpr int P2P_THREADS = 256;
constexpr int P2P_NC = 4;                            // 16-byte chunks per thread: 32 elements
constexpr int P2P_E = P2P_NC * FC_CHUNK;
constexpr int P2P_TILE = P2P_THREADS * P2P_E;
constexpr int P2P_STATUS_TIMEOUT = 1;
struct P2PArgs {
    const void* x[FC_MAX_P];          // EMU: rank p's input; else x[0] is this rank's
    void* y[FC_MAX_P];                // EMU: rank p's output; else y[0]
    QPtr s1[FC_MAX_P][FC_MAX_P];      // s1[p][c]: rank p's step-1 payload of chunk c
    QPtr s2[FC_MAX_P];                // s2[c]: owner c's step-2 payload of chunk c
    unsigned int* ctr1[FC_MAX_P];     // rank p's phase-1 counter
    unsigned int* ctr2[FC_MAX_P];     // rank p's phase-2 counter
    int* status;                      // OR-ed with P2P_STATUS_TIMEOUT on a wait that gave up
    size_t m;                         // chunk length in elements (n = P * m)
    int block;
    int rank;                         // this rank (ignored by EMU)
    int cpr;                          // CTAs per rank
    unsigned int epoch;               // k for the k-th call on the counters, or 0: derived from them
};

template <class T, int BITS, int P, bool EMU> cudaError_t launch_p2p(const P2PArgs& a, int grid, cudaStream_t st);
template <class T, int BITS, int P, bool EMU> cudaError_t p2p_max_ctas(int* ctas);

}  // namespace fc
