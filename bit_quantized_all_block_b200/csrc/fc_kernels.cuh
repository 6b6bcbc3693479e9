// fc_kernels.cuh -- sm_100a kernels of the two-step quantized all-reduce.
//
// k_quantize   step 1 on one rank            x_r -> step-1 payload
// k_rs         reduce-scatter (all chunks)   P step-1 payloads -> step-2 payload
// k_ag         all-gather dequantization     step-2 payload -> y
// k_fused      the whole all-reduce          P partials -> y (+ optional payloads)
//              (fc_fused.cuh)
//
// All four are HBM-bandwidth bound elementwise/reduction kernels (no dense
// contraction, so no tensor cores): persistent CTAs stride over tiles of
// FC_TILE elements, loads bypass L1, stores stream.  The fused kernel keeps
// every intermediate (step-1 codes, dequantized values, the fp32 sum, step-2
// codes) in registers; it writes payloads only when the caller asks for them.
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

// ---------------------------------------------------------------------------
// Step 1 on one rank.
template <class T, int BITS>
__global__ void __launch_bounds__(FC_THREADS) k_quantize(const QuantArgs a)
{
    __shared__ uint32_t red[FC_THREADS / 32];
    const Geo G = geometry(a.block);
    const T* x = static_cast<const T*>(a.x);
    for (size_t base = (size_t)blockIdx.x * FC_TILE; base < a.n; base += (size_t)gridDim.x * FC_TILE) {
        const size_t blk0 = base + (size_t)G.g * a.block;
        const bool valid = blk0 < a.n;
        const size_t e0 = base + (size_t)G.c0 * FC_CHUNK, e1 = base + (size_t)G.c1 * FC_CHUNK;
        uint4 r0 = make_uint4(0, 0, 0, 0), r1 = r0;
        if (valid) {
            r0 = ld_stream(x + e0);
            r1 = ld_stream(x + e1);
        }
        float mn, mx;
        chunk_minmax<T>(r0, r1, G.L, red, mn, mx);
        const BlockQ b = block_q<BITS>(mn, mx);
        float v[FC_ELEMS], sh[FC_ELEMS];
        widen16<T>(r0, r1, v);
#pragma unroll
        for (int i = 0; i < FC_ELEMS; i++)
            sh[i] = quant_shifted(v[i], b);
        if (valid) {
            store_codes<BITS>(a.out.codes, e0, sh);
            store_codes<BITS>(a.out.codes, e1, sh + 8);
            if (G.j == 0) {
                const size_t k = blk0 >> (__ffs(a.block) - 1);
                a.out.scales[k] = b.s;
                a.out.zps[k] = zp_byte(b);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Step 2 (reduce-scatter) for every chunk at once: chunk ownership does not
// change the arithmetic, since chunks are block-aligned and each block of the
// sum depends only on the same block of every rank.
template <int BITS, int P>
__global__ void __launch_bounds__(FC_THREADS) k_rs(const RsArgs a)
{
    __shared__ float2 red[FC_THREADS / 32];
    const Geo G = geometry(a.block);
    for (size_t base = (size_t)blockIdx.x * FC_TILE; base < a.n; base += (size_t)gridDim.x * FC_TILE) {
        const size_t blk0 = base + (size_t)G.g * a.block;
        const bool valid = blk0 < a.n;
        const size_t k = valid ? blk0 >> (__ffs(a.block) - 1) : 0;
        const size_t e0 = base + (size_t)G.c0 * FC_CHUNK, e1 = base + (size_t)G.c1 * FC_CHUNK;
        uint32_t w[P][2][2];
        float s[P];
        uint32_t z[P];
#pragma unroll
        for (int r = 0; r < P; r++) {
            if (valid) {
                load_codes<BITS>(a.in[r].codes, e0, w[r][0]);
                load_codes<BITS>(a.in[r].codes, e1, w[r][1]);
                s[r] = a.in[r].scales[k];
                z[r] = a.in[r].zps[k];
            } else {
                w[r][0][0] = w[r][0][1] = w[r][1][0] = w[r][1][1] = 0;
                s[r] = 1.0f;
                z[r] = 0;
            }
        }
        float acc[FC_ELEMS];
#pragma unroll
        for (int r = 0; r < P; r++) {
            const float mz = __uint_as_float(FC_MAGIC_BITS + z[r]);
            float sh[FC_ELEMS];
            unpack_chunk<BITS>(w[r][0], sh);
            unpack_chunk<BITS>(w[r][1], sh + 8);
#pragma unroll
            for (int i = 0; i < FC_ELEMS; i++) {
                const float xh = __fmul_rn(__fsub_rn(sh[i], mz), s[r]);
                acc[i] = (r == 0) ? xh : __fadd_rn(acc[i], xh);
            }
        }
        float mn = 0.0f, mx = 0.0f;
#pragma unroll
        for (int i = 0; i < FC_ELEMS; i++) {
            mn = fminf(mn, acc[i]);
            mx = fmaxf(mx, acc[i]);
        }
        group_minmax_f32(mn, mx, G.L, red);
        const BlockQ b = block_q<BITS>(mn, mx);
        float sh[FC_ELEMS];
#pragma unroll
        for (int i = 0; i < FC_ELEMS; i++)
            sh[i] = quant_shifted(acc[i], b);
        if (valid) {
            store_codes<BITS>(a.out.codes, e0, sh);
            store_codes<BITS>(a.out.codes, e1, sh + 8);
            if (G.j == 0) {
                a.out.scales[k] = b.s;
                a.out.zps[k] = zp_byte(b);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Step 3 (all-gather): dequantize to fp16/bf16.
template <class T, int BITS>
__global__ void __launch_bounds__(FC_THREADS) k_ag(const AgArgs a)
{
    const Geo G = geometry(a.block);
    T* y = static_cast<T*>(a.y);
    for (size_t base = (size_t)blockIdx.x * FC_TILE; base < a.n; base += (size_t)gridDim.x * FC_TILE) {
        const size_t blk0 = base + (size_t)G.g * a.block;
        if (blk0 >= a.n)
            continue;
        const size_t k = blk0 >> (__ffs(a.block) - 1);
        const size_t e0 = base + (size_t)G.c0 * FC_CHUNK, e1 = base + (size_t)G.c1 * FC_CHUNK;
        uint32_t w0[2], w1[2];
        load_codes<BITS>(a.in.codes, e0, w0);
        load_codes<BITS>(a.in.codes, e1, w1);
        const float s = a.in.scales[k];
        const float mz = __uint_as_float(FC_MAGIC_BITS + (uint32_t)a.in.zps[k]);
        float sh[FC_ELEMS], v[FC_ELEMS];
        unpack_chunk<BITS>(w0, sh);
        unpack_chunk<BITS>(w1, sh + 8);
#pragma unroll
        for (int i = 0; i < FC_ELEMS; i++)
            v[i] = __fmul_rn(__fsub_rn(sh[i], mz), s);
        st_stream(y + e0, narrow8<T>(v));
        st_stream(y + e1, narrow8<T>(v + 8));
    }
}

// Host-side launchers (one explicit instantiation per template in its .cu).
template <class T, int BITS> cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st);
template <int BITS, int P> cudaError_t launch_rs(const RsArgs& a, cudaStream_t st);
template <class T, int BITS> cudaError_t launch_ag(const AgArgs& a, cudaStream_t st);
template <class T, int B1, int B2, int P> cudaError_t launch_fused(const FusedArgs& a, cudaStream_t st);

// Persistent grid: enough CTAs of `threads` threads to fill every SM at the
// kernel's occupancy, never more than there are tiles of `tile` elements.
cudaError_t persistent_grid(const void* kernel, int threads, size_t n, size_t tile, int* grid);

}  // namespace fc
