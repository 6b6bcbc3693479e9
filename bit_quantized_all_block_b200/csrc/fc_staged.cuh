// fc_staged.cuh -- the staged kernels: the three steps of the two-step
// quantized all-reduce as separate launches with the payloads in HBM between
// them (Flash Communication, sciencestack.ai/paper/2412.04964: TL;DR, the
// quantize -> reduce-scatter -> all-gather structure; Fig. 5 right).
//
//   k_quantize<T, BITS, SPAN>   x_r -> step-1 payload (one rank)
//   k_rs<BITS, P>         P step-1 payloads -> step-2 payload (all chunks)
//   k_ag<T, BITS>         step-2 payload -> y
//
// Same layout as the fused kernel (fc_fused.cuh): 256-thread persistent CTAs,
// each thread owns E contiguous elements (one base pointer, immediate
// offsets, 128-bit accesses), a block is L = B/E consecutive threads that
// reduce min/max by xor-shuffles (and shared memory beyond a warp), the next
// tile's inputs are loaded as soon as the current ones are consumed, codes
// are rounded by one FMA, and the rarely binding upper clamp runs behind a
// warp-uniform branch.
#pragma once

#include "fc_fused.cuh"

namespace fc {

constexpr int ST_THREADS = 256;

template <int NC_>
struct StShape {
    static constexpr int NC = NC_;
    static constexpr int E = NC * FC_CHUNK;
    static constexpr int TILE = ST_THREADS * E;
};
using QuantShape = StShape<4>;                          // 32 elements per thread
using AgShape = StShape<4>;
// Reduce-scatter: 32 elements per thread and rank, except INT8 with more than
// four ranks (16), where 32 would hold 8 ranks x 8 code words in registers and
// cut the occupancy.
template <int BITS, int P> using RsShape = StShape<(BITS == 4 || P <= 4) ? 4 : 2>;

// Load a thread's E codes (E*BITS/8 contiguous bytes) at element offset e;
// WIDE: 32 bytes per load where there are 32 (codes 32-byte aligned).
template <int BITS, int NC, bool WIDE = false>
__device__ __forceinline__ void load_thread_codes(const uint8_t* codes, size_t e, uint32_t* w)
{
    constexpr int NW = NC * BITS / 4;
    const uint8_t* p = codes + e * BITS / 8;
    if constexpr (WIDE && NW % 8 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 8) {
            uint4 a, b;
            ld_nc_v8(p + 4 * i, a, b);
            w[i] = a.x;
            w[i + 1] = a.y;
            w[i + 2] = a.z;
            w[i + 3] = a.w;
            w[i + 4] = b.x;
            w[i + 5] = b.y;
            w[i + 6] = b.z;
            w[i + 7] = b.w;
        }
    } else if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 4) {
            const uint4 v = ld_nc(p + 4 * i);
            w[i] = v.x;
            w[i + 1] = v.y;
            w[i + 2] = v.z;
            w[i + 3] = v.w;
        }
    } else {
        const uint2 v = ld_stream_u2(p);
        w[0] = v.x;
        w[1] = v.y;
    }
}

// Shifted codes of chunk c of a thread's code words.
template <int BITS>
__device__ __forceinline__ void chunk_shifted(const uint32_t* w, int c, float* sh)
{
    if constexpr (BITS == 8)
        unpack_chunk<8>(w + 2 * c, sh);
    else
        unpack_chunk<4>(w + c, sh);
}

// Block extremes (0 folded in) of E fp32 values held by each of L threads.
// `red` alternates between two halves from tile to tile, so one barrier per
// tile separates every write from the reads of the previous use of its half.
template <int E>
__device__ __forceinline__ void block_minmax_f32(const float* v, int L, float2* red, float& mn, float& mx)
{
    mn = fminf(v[0], 0.0f);
    mx = fmaxf(v[0], 0.0f);
#pragma unroll
    for (int i = 1; i + 1 < E; i += 2) {
        mn = min3(mn, v[i], v[i + 1]);
        mx = max3(mx, v[i], v[i + 1]);
    }
    mn = fminf(mn, v[E - 1]);
    mx = fmaxf(mx, v[E - 1]);
    group_minmax_f32<false>(mn, mx, L, red);
}

// Quantize E fp32 values (one thread's share of a block) and store codes,
// scale and zero-point.
template <int BITS, int NC, bool CLAMP>
__device__ __forceinline__ void quant_store(const float* v, const BlockQ& b, const QPtr& out, size_t e,
                                            bool leader, size_t k)
{
    const float cqz = __fsub_rn(b.cq, b.zf);
    const uint32_t offset = pack_offset<BITS>(b);
    const float2 inv2 = dup2(b.inv), m2 = dup2(FC_MAGIC);
    uint32_t words[NC * BITS / 4];
#pragma unroll
    for (int c = 0; c < NC; c++) {
        float r[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            st2(r, i, fma2(ld2(v, c * 8 + i), inv2, m2));   // FC_MAGIC + rne(v*inv)
        if (CLAMP) {
#pragma unroll
            for (int i = 0; i < 8; i++)
                r[i] = fminf(r[i], cqz);
        }
        pack_shifted<BITS>(r, b, offset, words, c);
    }
    store_thread_codes<BITS, NC>(out.codes, e, words);
    if (leader) {
        out.scales[k] = b.s;
        out.zps[k] = zp_byte(b);
    }
}

// ---------------------------------------------------------------------------
// Step 1 on one rank.  SPAN (blocks that span warps, reduced through shared
// memory and a CTA barrier; the launcher selects it for blocks above 32*E):
// the next tile's loads are issued before the block's reduction, so they are
// in flight during the barrier -- 8 % faster at blocks of 4096.  Within a warp
// (shuffles only) the loads wait until the scales are known, which measured
// 1-2 % faster at blocks of 128.
template <class T, int BITS, bool SPAN>
__global__ void __launch_bounds__(ST_THREADS) k_quantize(const QuantArgs a)
{
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
    constexpr int NC = QuantShape::NC, E = QuantShape::E, TILE = QuantShape::TILE;
    __shared__ uint32_t red[2][ST_THREADS / 32];   // alternating halves: one barrier per tile
    const int L = a.block / E;
    const int j = threadIdx.x % L;
    const int lg_block = __ffs(a.block) - 1;
    const size_t toff = (size_t)threadIdx.x * E;
    const size_t stride = (size_t)gridDim.x * TILE;
    const T* x = static_cast<const T*>(a.x);

    uint4 raw[NC];
    {
        const size_t e0 = (size_t)blockIdx.x * TILE + toff;
        if (e0 < a.n) {
            load_chunks<T, NC>(raw, x + e0);
        } else {
#pragma unroll
            for (int c = 0; c < NC; c++)
                raw[c] = make_uint4(0, 0, 0, 0);
        }
    }
    int half = 0;
    for (size_t base = (size_t)blockIdx.x * TILE; base < a.n; base += stride, half ^= 1) {
        const size_t e = base + toff;
        const bool valid = e < a.n;
        const size_t k = e >> lg_block;
        const uint32_t own = local_min_negmax<T, NC>(raw);
        float v[E];
        BlockQ b;
        bool clamp;
        const auto scales = [&] {
            const T2 t = as_t2<T2>(group_min_negmax<T, false>(own, L, red[half]));
            const float mx = fmaxf(-P2::hi(t), 0.0f);
            b = block_q<BITS>(fminf(P2::lo(t), 0.0f), mx);
            clamp = __any_sync(0xffffffffu, top_code_overflows(mx, b));
        };
        const auto widen_and_refill = [&] {
#pragma unroll
            for (int c = 0; c < NC; c++) {
                const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    const float2 f = P2::to_f2(as_t2<T2>(w[h]));
                    v[c * 8 + 2 * h] = f.x;
                    v[c * 8 + 2 * h + 1] = f.y;
                }
            }
            if (e + stride < a.n)
                load_chunks<T, NC>(raw, x + e + stride);
        };
        if constexpr (SPAN) {
            widen_and_refill();
            scales();
        } else {
            scales();
            widen_and_refill();
        }
        if (valid) {
            if (clamp)
                quant_store<BITS, NC, true>(v, b, a.out, e, j == 0, k);
            else
                quant_store<BITS, NC, false>(v, b, a.out, e, j == 0, k);
        }
    }
}

// ---------------------------------------------------------------------------
// Step 2 (reduce-scatter) for every chunk at once: chunk ownership does not
// change the arithmetic, since chunks are block-aligned and each block of the
// sum depends only on the same block of every rank.
template <int BITS, int P>
__global__ void __launch_bounds__(ST_THREADS) k_rs(const RsArgs a)
{
    constexpr int NC = RsShape<BITS, P>::NC, E = RsShape<BITS, P>::E, TILE = RsShape<BITS, P>::TILE;
    constexpr int NW = NC * BITS / 4;
    __shared__ float2 red[2][ST_THREADS / 32];     // alternating halves: one barrier per tile
    const int L = a.block / E;
    const int j = threadIdx.x % L;
    const int lg_block = __ffs(a.block) - 1;
    const size_t toff = (size_t)threadIdx.x * E;
    const size_t stride = (size_t)gridDim.x * TILE;

    uint32_t w[P][NW];
    float s[P], mz[P];
    {
        const size_t e0 = (size_t)blockIdx.x * TILE + toff;
        const size_t k0 = e0 >> lg_block;
#pragma unroll
        for (int r = 0; r < P; r++) {
            if (e0 < a.n) {
                load_thread_codes<BITS, NC>(a.in[r].codes, e0, w[r]);
                s[r] = a.in[r].scales[k0];
                mz[r] = __uint_as_float(FC_MAGIC_BITS + a.in[r].zps[k0]);
            } else {
#pragma unroll
                for (int i = 0; i < NW; i++)
                    w[r][i] = 0;
                s[r] = 1.0f;
                mz[r] = FC_MAGIC;
            }
        }
    }
    int half = 0;
    for (size_t base = (size_t)blockIdx.x * TILE; base < a.n; base += stride, half ^= 1) {
        const size_t e = base + toff;
        const bool valid = e < a.n;
        const bool valid_next = e + stride < a.n;
        const size_t k = e >> lg_block;
        const size_t kn = (e + stride) >> lg_block;
        float acc[E];
#pragma unroll
        for (int r = 0; r < P; r++) {
            const float2 nmz2 = dup2(-mz[r]), s2 = dup2(s[r]);
#pragma unroll
            for (int c = 0; c < NC; c++) {
                float sh[8];
                chunk_shifted<BITS>(w[r], c, sh);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float2 xh = prod2(add2(ld2(sh, i), nmz2), s2);    // (q - z) * s
                    st2(acc, c * 8 + i, (r == 0) ? xh : add2(ld2(acc, c * 8 + i), xh));
                }
            }
            if (valid_next) {   // refill rank r with the next tile
                load_thread_codes<BITS, NC>(a.in[r].codes, e + stride, w[r]);
                s[r] = a.in[r].scales[kn];
                mz[r] = __uint_as_float(FC_MAGIC_BITS + a.in[r].zps[kn]);
            }
        }
        float mn, mx;
        block_minmax_f32<E>(acc, L, red[half], mn, mx);
        const BlockQ b = block_q<BITS>(mn, mx);
        const bool clamp = __any_sync(0xffffffffu, top_code_overflows(mx, b));
        if (valid) {
            if (clamp)
                quant_store<BITS, NC, true>(acc, b, a.out, e, j == 0, k);
            else
                quant_store<BITS, NC, false>(acc, b, a.out, e, j == 0, k);
        }
    }
}

// ---------------------------------------------------------------------------
// Step 3 (all-gather): dequantize to fp16/bf16.  WIDE: 32-byte stores of y
// and (INT8) 32-byte code loads; y and the codes 32-byte aligned.  The next
// tile's codes, scale and zero-point are loaded before the current tile is
// dequantized and stored.
template <class T, int BITS, bool WIDE>
__global__ void __launch_bounds__(ST_THREADS) k_ag(const AgArgs a)
{
    constexpr int NC = AgShape::NC, E = AgShape::E, TILE = AgShape::TILE;
    constexpr int NW = NC * BITS / 4;
    const int lg_block = __ffs(a.block) - 1;
    const size_t toff = (size_t)threadIdx.x * E;
    const size_t stride = (size_t)gridDim.x * TILE;
    T* y = static_cast<T*>(a.y);

    uint32_t w[NW];
    float s = 1.0f, mz = FC_MAGIC;
    size_t e = (size_t)blockIdx.x * TILE + toff;
    if (e < a.n) {
        load_thread_codes<BITS, NC, WIDE>(a.in.codes, e, w);
        s = a.in.scales[e >> lg_block];
        mz = __uint_as_float(FC_MAGIC_BITS + a.in.zps[e >> lg_block]);
    }
    for (; e < a.n + toff; e += stride) {   // every thread of the CTA runs the same trip count
        const size_t en = e + stride;
        uint32_t wn[NW];
        float sn = 1.0f, mzn = FC_MAGIC;
        if (en < a.n) {
            load_thread_codes<BITS, NC, WIDE>(a.in.codes, en, wn);
            sn = a.in.scales[en >> lg_block];
            mzn = __uint_as_float(FC_MAGIC_BITS + a.in.zps[en >> lg_block]);
        }
        if (e < a.n) {
            const float2 nmz2 = dup2(-mz), s2 = dup2(s);
            uint4 ov[NC];
#pragma unroll
            for (int c = 0; c < NC; c++) {
                float sh[8], v[8];
                chunk_shifted<BITS>(w, c, sh);
#pragma unroll
                for (int i = 0; i < 8; i += 2)
                    st2(v, i, mul2(add2(ld2(sh, i), nmz2), s2));
                ov[c] = narrow8<T>(v);
            }
            store_chunks<NC, WIDE>(y + e, ov);
        }
#pragma unroll
        for (int i = 0; i < NW; i++)
            w[i] = wn[i];
        s = sn;
        mz = mzn;
    }
}

}  // namespace fc
