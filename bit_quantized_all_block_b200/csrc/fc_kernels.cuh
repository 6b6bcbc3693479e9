// fc_kernels.cuh -- argument blocks and launchers of the sm_100a kernels of
// the two-step quantized all-reduce:
//
// k_quantize   step 1 on one rank            x_r -> step-1 payload        (fc_staged.cuh)
// k_rs         reduce-scatter (all chunks)   P step-1 payloads -> step-2  (fc_staged.cuh)
// k_ag         all-gather dequantization     step-2 payload -> y          (fc_staged.cuh)
// k_fused      the whole all-reduce          P partials -> y (+ payloads) (fc_fused.cuh)
//
// All four are HBM-bandwidth bound elementwise/reduction kernels (no dense
// contraction, so no tensor cores): persistent CTAs stride over tiles, loads
// are 128-bit, stores stream.  The fused kernel keeps every intermediate
// (step-1 codes, dequantized values, the fp32 sum, step-2 codes) in
// registers; it writes payloads only when the caller asks for them.
#pragma once

#include "fc_device.cuh"

namespace fc {

constexpr int FC_MAX_P = 8;

struct QPtr {
    uint8_t* codes;
    float* scales;
    uint8_t* zps;
};

struct QuantArgs {
    const void* x;
    QPtr out;
    size_t n;
    int block;
};

struct RsArgs {
    QPtr in[FC_MAX_P];
    QPtr out;
    size_t n;
    int block;
};

struct AgArgs {
    QPtr in;
    void* y;
    size_t n;
    int block;
};

struct FusedArgs {
    const void* x[FC_MAX_P];
    QPtr step1[FC_MAX_P];
    QPtr step2;
    void* y;
    size_t n;
    int block;
    int write_step1;
    int write_step2;
};

// Host-side launchers (one explicit instantiation per template in its .cu).
template <class T, int BITS> cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st);
template <int BITS, int P> cudaError_t launch_rs(const RsArgs& a, cudaStream_t st);
template <class T, int BITS, bool WIDE = false> cudaError_t launch_ag(const AgArgs& a, cudaStream_t st);
template <class T, int B1, int B2, int P, bool SMALL = false, bool WIDE = false, bool SPLIT = true>
cudaError_t launch_fused(const FusedArgs& a, cudaStream_t st);

// Elements per thread per rank of the fused kernel's bandwidth and latency
// shapes.  A block is L = block / E threads; the lane-split scale form (SPLIT)
// needs min(L, 32) >= P.
constexpr int FC_FUSED_E = 16;
constexpr int FC_FUSED_SMALL_E = 8;
inline bool fused_lane_split(int block, int P, bool small)
{
    const int L = block / (small ? FC_FUSED_SMALL_E : FC_FUSED_E);
    return (L < 32 ? L : 32) >= P;
}

// SMs of the current device and co-resident CTAs of `kernel` per SM at
// `threads` threads (queried once per device, kernel and thread count).
cudaError_t kernel_residency(const void* kernel, int threads, int* sms, int* per_sm);

// Persistent grid: enough CTAs of `threads` threads to fill every SM at the
// kernel's occupancy, never more than there are tiles of `tile` elements.
cudaError_t persistent_grid(const void* kernel, int threads, size_t n, size_t tile, int* grid);

}  // namespace fc
