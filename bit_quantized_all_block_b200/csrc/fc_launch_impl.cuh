// fc_launch_impl.cuh -- launcher bodies, included by the instantiation units.
#pragma once

#include "fc_staged.cuh"

namespace fc {

template <class T, int BITS, bool SPAN>
cudaError_t launch_quantize_as(const QuantArgs& a, cudaStream_t st)
{
    int grid = 0;
    cudaError_t e = persistent_grid((const void*)k_quantize<T, BITS, SPAN>, ST_THREADS, a.n, QuantShape::TILE, &grid);
    if (e != cudaSuccess)
        return e;
    k_quantize<T, BITS, SPAN><<<grid, ST_THREADS, 0, st>>>(a);
    return cudaGetLastError();
}

template <class T, int BITS>
cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st)
{
    // blocks wider than a warp's 32 threads reduce through shared memory
    return a.block > 32 * QuantShape::E ? launch_quantize_as<T, BITS, true>(a, st)
                                         : launch_quantize_as<T, BITS, false>(a, st);
}

template <int BITS, int P>
cudaError_t launch_rs(const RsArgs& a, cudaStream_t st)
{
    int grid = 0;
    cudaError_t e = persistent_grid((const void*)k_rs<BITS, P>, ST_THREADS, a.n, RsShape<BITS, P>::TILE, &grid);
    if (e != cudaSuccess)
        return e;
    k_rs<BITS, P><<<grid, ST_THREADS, 0, st>>>(a);
    return cudaGetLastError();
}

template <class T, int BITS, bool WIDE>
cudaError_t launch_ag(const AgArgs& a, cudaStream_t st)
{
    int grid = 0;
    cudaError_t e = persistent_grid((const void*)k_ag<T, BITS, WIDE>, ST_THREADS, a.n, AgShape::TILE, &grid);
    if (e != cudaSuccess)
        return e;
    k_ag<T, BITS, WIDE><<<grid, ST_THREADS, 0, st>>>(a);
    return cudaGetLastError();
}

template <class T, int B1, int B2, int P, bool SMALL, bool WIDE, bool SPLIT>
cudaError_t launch_fused(const FusedArgs& a, cudaStream_t st)
{
    using S = FuShape<P, SMALL>;
    static_assert(S::E == (SMALL ? FC_FUSED_SMALL_E : FC_FUSED_E), "fused_lane_split() assumes this shape");
    int grid = 0;
    cudaError_t e =
        persistent_grid((const void*)k_fused<T, B1, B2, P, SMALL, WIDE, SPLIT>, S::THREADS, a.n, S::TILE, &grid);
    if (e != cudaSuccess)
        return e;
    k_fused<T, B1, B2, P, SMALL, WIDE, SPLIT><<<grid, S::THREADS, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace fc
