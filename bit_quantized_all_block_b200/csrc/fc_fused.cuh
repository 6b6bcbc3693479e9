// fc_fused.cuh -- the fused two-step quantized all-reduce kernel (sm_100a).
//
// One pass per block index k: load block k of all P ranks, quantize and
// dequantize each (step 1), sum the dequantized values in rank order (the
// reduce-scatter), requantize and dequantize the sum (step 2) and store the
// fp16/bf16 result (the all-gather); the wire payloads are written only when
// the caller asks for them.  Flash Communication (sciencestack.ai/paper/
// 2412.04964), TL;DR: the method is implemented as one fused CUDA kernel.
//
// The kernel moves ~1 GB per call on the 70B-shaped workload; with about a dozen
// operations per input element it would be bound by instruction issue as much
// as by HBM, so it is laid out to cut instructions (after which it waits on
// its loads rather than on issue):
//  * thread t of a CTA owns E = 16 contiguous elements of every rank in the
//    tile (8 in the latency shape); a block of B elements is L = B/E
//    consecutive threads, so a 128-block needs 8 threads and 3 shuffle
//    rounds.  All loads and stores of a thread use one base pointer with
//    immediate offsets; a thread's 32 bytes of a rank move as one 32-byte
//    access when the buffers allow it (WIDE), else as two 16-byte ones;
//  * the P per-rank scale computations of a block are spread over the lanes
//    of its group (lane r computes rank r, whose block extremes reach it by a
//    reduce-scatter over the group's lanes) and broadcast with shuffles;
//  * the upper code clamp binds only when the block maximum's code rounds to
//    qmax + 1 -- rare -- so it is checked once per block from the maximum
//    and applied behind a warp-uniform branch around the per-element minimum
//    only, so each body exists once (the rank loop is unrolled P times and
//    its code size shows up as instruction-fetch stalls); the lower clamp
//    never binds (see the lower-clamp note in fc_device.cuh);
//    that lane-split form is used whenever a block's thread group has at
//    least P lanes (SPLIT, chosen by the host from the block size; narrower
//    groups compute every rank's scale in every lane), so the unrolled loop
//    carries only one form;
//  * each rank's registers are refilled with the next tile's data as soon as
//    that rank is consumed, so loads stay in flight during the rest of the
//    tile (software pipelining without extra registers);
//  * code bytes are formed only when a payload is written;
//  * the per-element floating-point chains run on packed fp32 pairs (see the
//    contraction note in fc_device.cuh for how the rank-order sum is kept
//    exact).
#pragma once

#include "fc_kernels.cuh"

namespace fc {

constexpr int FU_THREADS = 256;

#ifndef FC_FUSED_NC_SMALL_P
#define FC_FUSED_NC_SMALL_P 2
#endif
#ifndef FC_FUSED_MIN_CTAS
#define FC_FUSED_MIN_CTAS 2
#endif

// Launch shape.  The bandwidth shape (SMALL = false): 256-thread CTAs, two CTAs
// per SM, 16 elements per thread per rank.  The latency shape for
// decode-sized messages (SMALL = true): 64-thread CTAs with 8 elements per
// thread per rank, so a call of a few hundred KB spreads over many more SMs
// and each thread's dependent chain is half as long; it serves blocks of up to
// 256 elements (a block must fit in one warp: 32 threads x 8).
template <int P, bool SMALL = false>
struct FuShape {
    static constexpr int THREADS = SMALL ? 64 : FU_THREADS;
    static constexpr int NC = SMALL ? 1 : (P <= 4 ? FC_FUSED_NC_SMALL_P : 2);  // 16-byte chunks per thread per rank
    static constexpr int E = NC * FC_CHUNK;                       // elements per thread per rank
    static constexpr int TILE = THREADS * E;                      // elements per rank per tile
    static constexpr int MIN_CTAS = SMALL ? 8 : FC_FUSED_MIN_CTAS;
};

__device__ __forceinline__ uint4 ld_nc(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float min3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// In-thread {min, -max} of the fp16/bf16 values of NC chunks.
template <class T, int NC>
__device__ __forceinline__ uint32_t local_min_negmax(const uint4* c)
{
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
    T2 m = as_t2<T2>(c[0].x), M = m;
#pragma unroll
    for (int i = 0; i < NC; i++) {
        const uint32_t w[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
#pragma unroll
        for (int k = (i == 0 ? 1 : 0); k < 4; k++) {
            m = __hmin2(m, as_t2<T2>(w[k]));
            M = __hmax2(M, as_t2<T2>(w[k]));
        }
    }
    const T2 nM = __hneg2(M);
    return t2_bits(__hmin2(P2::lows(m, nM), P2::highs(m, nM)));
}

// Whether the largest code of a block, rne(mx*inv) + z, exceeds qmax.
__device__ __forceinline__ bool top_code_overflows(float mx, const BlockQ& b)
{
    return __fadd_rn(round_product_shifted(mx, b.inv), b.zf) > b.cq;
}

// Store a thread's E codes (E*BITS/8 contiguous bytes) at element offset e.
template <int BITS, int NC>
__device__ __forceinline__ void store_thread_codes(uint8_t* codes, size_t e, const uint32_t* w)
{
    constexpr int NW = NC * BITS / 4;   // 32-bit words: INT8 2 per chunk, INT4 1 per chunk
    uint8_t* p = codes + e * BITS / 8;
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 4)
            st_stream(p + 4 * i, make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]));
    } else if constexpr (NW == 2) {
        st_stream(p, make_uint2(w[0], w[1]));
    } else {
        st_stream(p, w[0]);
    }
}

// Step-1 work on one rank's values: quantize, dequantize, accumulate in rank
// order; optionally store codes, scale and zero-point.  `clamp` (warp-uniform)
// says whether any block of the warp needs the upper code clamp; the branch
// skips the per-element minimum in the usual case without a second copy of
// the body (the rank loop is unrolled P times, so code size matters).
template <class T, int BITS, int NC, bool FIRST>
__device__ __forceinline__ void rank_body(const uint4* raw, const BlockQ& b, bool clamp, float* acc, bool store,
                                          const QPtr& out, size_t e, bool leader, size_t k)
{
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
    const float2 inv2 = dup2(b.inv), m2 = dup2(FC_MAGIC), nm2 = dup2(-FC_MAGIC), s2 = dup2(b.s);
    uint32_t words[NC * BITS / 4];
#pragma unroll
    for (int c = 0; c < NC; c++) {
        const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
        float r[8];
#pragma unroll
        for (int h = 0; h < 4; h++)
            st2(r, 2 * h, fma2(P2::to_f2(as_t2<T2>(w[h])), inv2, m2));   // FC_MAGIC + rne(v*inv)
        if (clamp) {
            const float cqz = __fsub_rn(b.cq, b.zf);   // FC_MAGIC + qmax - z (exact)
#pragma unroll
            for (int i = 0; i < 8; i++)
                r[i] = fminf(r[i], cqz);
        }
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float2 xh = mul2(add2(ld2(r, i), nm2), s2);              // (q - z) * s
            if (FIRST)
                st2(acc, c * 8 + i, xh);
            else
                acc_add(acc, c * 8 + i, xh);
        }
        if (store)
            pack_shifted<BITS>(r, b, pack_offset<BITS>(b), words, c);
    }
    if (store) {
        store_thread_codes<BITS, NC>(out.codes, e, words);
        if (leader) {
            out.scales[k] = b.s;
            out.zps[k] = zp_byte(b);
        }
    }
}

// Step 2 on the sums: requantize, dequantize, store y (+ payload); `clamp`
// as for rank_body.
template <class T, int BITS, int NC, bool WIDE>
__device__ __forceinline__ void sum_body(const float* acc, const BlockQ& b, bool clamp, T* y, bool store,
                                         const QPtr& out, size_t e, bool leader, size_t k)
{
    const float2 inv2 = dup2(b.inv), m2 = dup2(FC_MAGIC), nm2 = dup2(-FC_MAGIC), s2 = dup2(b.s);
    uint32_t words[NC * BITS / 4];
    uint4 ov[NC];
#pragma unroll
    for (int c = 0; c < NC; c++) {
        float r[8], o[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            st2(r, i, fma2(ld2(acc, c * 8 + i), inv2, m2));
        if (clamp) {
            const float cqz = __fsub_rn(b.cq, b.zf);
#pragma unroll
            for (int i = 0; i < 8; i++)
                r[i] = fminf(r[i], cqz);
        }
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            st2(o, i, mul2(add2(ld2(r, i), nm2), s2));
        if constexpr (WIDE)
            ov[c] = narrow8<T>(o);
        else
            st_stream(y + e + c * FC_CHUNK, narrow8<T>(o));
        if (store)
            pack_shifted<BITS>(r, b, pack_offset<BITS>(b), words, c);
    }
    if constexpr (WIDE)
        store_chunks<NC, true>(y + e, ov);
    if (store) {
        store_thread_codes<BITS, NC>(out.codes, e, words);
        if (leader) {
            out.scales[k] = b.s;
            out.zps[k] = zp_byte(b);
        }
    }
}

__device__ __forceinline__ BlockQ shfl_blockq(const BlockQ& mine, int src, float cq)
{
    BlockQ b;
    b.s = __shfl_sync(0xffffffffu, mine.s, src);
    b.inv = __shfl_sync(0xffffffffu, mine.inv, src);
    b.mz = __shfl_sync(0xffffffffu, mine.mz, src);
    b.zf = __fsub_rn(b.mz, FC_MAGIC);
    b.cq = cq;
    return b;
}

// Load NC chunks at p; WIDE: in pairs, one 32-byte load each (p 32-byte aligned).
template <class T, int NC, bool WIDE = false>
__device__ __forceinline__ void load_chunks(uint4* raw, const T* p)
{
    if constexpr (WIDE && NC % 2 == 0) {
#pragma unroll
        for (int c = 0; c < NC; c += 2)
            ld_nc_v8(p + c * FC_CHUNK, raw[c], raw[c + 1]);
    } else {
#pragma unroll
        for (int c = 0; c < NC; c++)
            raw[c] = ld_nc(p + c * FC_CHUNK);
    }
}

// Unquantized step 1 (16-bit values sent as they are): the reduce-scatter sums
// the exactly widened inputs.
template <class T, int NC, bool FIRST>
__device__ __forceinline__ void rank_body_plain(const uint4* raw, float* acc)
{
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
#pragma unroll
    for (int c = 0; c < NC; c++) {
        const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
        for (int h = 0; h < 4; h++) {
            const float2 v = P2::to_f2(as_t2<T2>(w[h]));
            const int i = c * 8 + 2 * h;
            st2(acc, i, FIRST ? v : add2(ld2(acc, i), v));
        }
    }
}

// B1 / B2: bits of the reduce-scatter and of the all-gather step, each 4, 8
// or 16 (16 = that step sends fp16/bf16 values unquantized; Fig. 5 right of
// the page compares quantizing before RS with quantizing before AG).
// WIDE: inputs and output are moved with 32-byte accesses (every x[r] and y
// 32-byte aligned; NC even).  SPLIT: see the step-1 scales below.
template <class T, int B1, int B2, int P, bool SMALL = false, bool WIDE = false, bool SPLIT = true>
__global__ void __launch_bounds__(FuShape<P, SMALL>::THREADS, FuShape<P, SMALL>::MIN_CTAS)
    k_fused(const FusedArgs a)
{
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
    using S = FuShape<P, SMALL>;
    constexpr int NC = S::NC, E = S::E, TILE = S::TILE;
    constexpr int QB1 = B1 == 16 ? 8 : B1;     // (unused when B1 == 16)
    __shared__ uint32_t red16[P][S::THREADS / 32];
    __shared__ float2 red32[S::THREADS / 32];

    const int L = a.block / E;                 // threads per block (1 .. 256)
    const int j = threadIdx.x % L;             // member index inside the block
    const int Lw = L < 32 ? L : 32;            // threads of the block inside this warp
    const int lane = threadIdx.x & 31;
    const int grp = lane & ~(Lw - 1);          // first lane of my group in the warp
    // SPLIT: lane r of a block's group computes rank r's scale (the host
    // selects this form only when the group has at least P lanes); otherwise
    // every lane computes every rank's scale.  A compile-time choice keeps the
    // unused form out of the unrolled rank loop.
    constexpr bool split = SPLIT;
    const size_t toff = (size_t)threadIdx.x * E;
    const size_t stride = (size_t)gridDim.x * TILE;
    const float cq1 = __uint_as_float(FC_MAGIC_BITS + (uint32_t)((1 << QB1) - 1));

    const int lg_block = __ffs(a.block) - 1;   // block is a power of two

    uint4 raw[P][NC];
    {
        const size_t e0 = (size_t)blockIdx.x * TILE + toff;
#pragma unroll
        for (int r = 0; r < P; r++) {
            if (e0 < a.n) {
                load_chunks<T, NC, WIDE>(raw[r], static_cast<const T*>(a.x[r]) + e0);
            } else {
#pragma unroll
                for (int c = 0; c < NC; c++)
                    raw[r][c] = make_uint4(0, 0, 0, 0);
            }
        }
    }
    for (size_t base = (size_t)blockIdx.x * TILE; base < a.n; base += stride) {
        // My elements [e, e + E) lie inside one block; it is valid iff e < n
        // (blocks never straddle n because n is a multiple of the block).
        const size_t e = base + toff;
        const bool valid = e < a.n;
        const bool valid_next = e + stride < a.n;
        const size_t k = e >> lg_block;
        const bool leader = valid && j == 0;
        float acc[E];

        if constexpr (B1 == 16) {
#pragma unroll
            for (int r = 0; r < P; r++) {
                if (r == 0)
                    rank_body_plain<T, NC, true>(raw[r], acc);
                else
                    rank_body_plain<T, NC, false>(raw[r], acc);
                if (valid_next)
                    load_chunks<T, NC, WIDE>(raw[r], static_cast<const T*>(a.x[r]) + e + stride);
            }
        } else {
            // ---- block extremes of every rank (packed {min, -max}) ---------
            uint32_t u[P];
#pragma unroll
            for (int r = 0; r < P; r++)
                u[r] = local_min_negmax<T, NC>(raw[r]);
            // With more than four ranks the lane-split form gathers each lane's
            // one rank by a reduce-scatter (below); otherwise all-reduce every
            // rank over the group (at P <= 4 the reduce-scatter's selects cost
            // more than its saved shuffles: the 70B-shaped INT8 kernel was 2 %
            // slower with it).
            constexpr bool scatter = split && P > 4;
            if constexpr (!scatter) {
                for (int o = 1; o < Lw; o <<= 1) {
#pragma unroll
                    for (int r = 0; r < P; r++)
                        u[r] = t2_bits(
                            __hmin2(as_t2<T2>(u[r]), as_t2<T2>(__shfl_xor_sync(0xffffffffu, u[r], o))));
                }
            }
            // ---- step-1 scales: one lane per rank when the group is wide enough
            BlockQ mine;
            bool clamp1 = false;
            if constexpr (split) {
                // Lane `me` of the group computes one rank's scale: rank me
                // (lanes past P: rank 0) after the all-reduce; with the
                // reduce-scatter, rank (me mod PW), PW = P rounded up to a power
                // of two (ranks past P stand for rank 0).  The reduce-scatter is
                // recursive halving over the lane bits below PW: at offset h a
                // lane keeps the upper half of its remaining ranks if its bit h
                // is set, else the lower half, and takes the partner's values of
                // the half it keeps, which leaves lane me with rank (me mod PW)
                // over the PW lanes that share its higher bits (PW - 1 exchanges
                // instead of P per round of an all-reduce); the rest of the
                // group then reduces that one value.
                constexpr int PW = P <= 1 ? 1 : P <= 2 ? 2 : P <= 4 ? 4 : 8;
                const int me = lane - grp;
                const int rr = scatter ? ((me & (PW - 1)) < P ? (me & (PW - 1)) : 0) : (me < P ? me : 0);
                uint32_t um = u[0];
                if constexpr (scatter) {
                    uint32_t v[PW];
#pragma unroll
                    for (int r = 0; r < PW; r++)
                        v[r] = u[r < P ? r : 0];
#pragma unroll
                    for (int h = PW / 2; h >= 1; h >>= 1) {
                        const bool up = (lane & h) != 0;
#pragma unroll
                        for (int i = 0; i < h; i++) {
                            const uint32_t keep = up ? v[i + h] : v[i];
                            const uint32_t send = up ? v[i] : v[i + h];
                            v[i] = t2_bits(
                                __hmin2(as_t2<T2>(keep), as_t2<T2>(__shfl_xor_sync(0xffffffffu, send, h))));
                        }
                    }
                    um = v[0];
                    for (int o = PW; o < Lw; o <<= 1)
                        um = t2_bits(__hmin2(as_t2<T2>(um), as_t2<T2>(__shfl_xor_sync(0xffffffffu, um, o))));
                } else if (L <= 32) {
#pragma unroll
                    for (int r = 1; r < P; r++)
                        um = (rr == r) ? u[r] : um;
                }
                if (L > 32) {                   // blocks that span warps: the group is the warp
                    if constexpr (scatter) {
                        if (me < P)
                            red16[me][threadIdx.x >> 5] = um;
                    } else if (lane == 0) {
#pragma unroll
                        for (int r = 0; r < P; r++)
                            red16[r][threadIdx.x >> 5] = u[r];
                    }
                    __syncthreads();
                    const int nw = L >> 5, w0 = (threadIdx.x / L) * nw;
                    um = red16[rr][w0];
                    for (int i = 1; i < nw; i++)
                        um = t2_bits(__hmin2(as_t2<T2>(um), as_t2<T2>(red16[rr][w0 + i])));
                    // With both steps quantized, the step-2 reduction's barrier
                    // separates these reads from the next tile's writes.
                    if (B2 == 16)
                        __syncthreads();
                }
                const T2 t = as_t2<T2>(um);
                const float mx = fmaxf(-P2::hi(t), 0.0f);
                mine = block_q<QB1>(fminf(P2::lo(t), 0.0f), mx);
                clamp1 = __any_sync(0xffffffffu, top_code_overflows(mx, mine));
            }
            // (without SPLIT the group is narrower than P lanes, so L < 32 and
            // every lane holds every rank's extremes in u; with SPLIT lane r
            // of the group holds rank r's scale, fetched by shfl_blockq below)

            const bool store1 = a.write_step1 && valid;
#pragma unroll
            for (int r = 0; r < P; r++) {
                BlockQ b;
                bool clamp = clamp1;
                if constexpr (split) {
                    b = shfl_blockq(mine, grp + r, cq1);
                } else {
                    const T2 t = as_t2<T2>(u[r]);
                    const float mx = fmaxf(-P2::hi(t), 0.0f);
                    b = block_q<QB1>(fminf(P2::lo(t), 0.0f), mx);
                    clamp = __any_sync(0xffffffffu, top_code_overflows(mx, b));
                }
                if (r == 0)
                    rank_body<T, QB1, NC, true>(raw[r], b, clamp, acc, store1, a.step1[r], e, leader, k);
                else
                    rank_body<T, QB1, NC, false>(raw[r], b, clamp, acc, store1, a.step1[r], e, leader, k);
                if (valid_next)   // refill rank r with the next tile while this one finishes
                    load_chunks<T, NC, WIDE>(raw[r], static_cast<const T*>(a.x[r]) + e + stride);
            }
        }

        T* y = static_cast<T*>(a.y);
        if constexpr (B2 == 16) {
            // ---- unquantized all-gather: the sum rounded to fp16/bf16 ----------
            if (valid) {
                uint4 ov[NC];
#pragma unroll
                for (int c = 0; c < NC; c++)
                    ov[c] = narrow8<T>(acc + c * FC_CHUNK);
                store_chunks<NC, WIDE>(y + e, ov);
            }
        } else {
            // ---- step 2: requantize the sum -------------------------------------
            float mn = fminf(acc[0], 0.0f), mx = fmaxf(acc[0], 0.0f);
#pragma unroll
            for (int i = 1; i + 1 < E; i += 2) {
                mn = min3(mn, acc[i], acc[i + 1]);
                mx = max3(mx, acc[i], acc[i + 1]);
            }
            mn = fminf(mn, acc[E - 1]);
            mx = fmaxf(mx, acc[E - 1]);
            // the next tile's step-1 barrier separates these reads from the next writes
            group_minmax_f32<B1 == 16>(mn, mx, L, red32);
            const BlockQ b2 = block_q<B2>(mn, mx);
            const bool clamp2 = __any_sync(0xffffffffu, top_code_overflows(mx, b2));
            if (valid)
                sum_body<T, B2, NC, WIDE>(acc, b2, clamp2, y, a.write_step2 != 0, a.step2, e, leader, k);
        }
    }
}

}  // namespace fc
