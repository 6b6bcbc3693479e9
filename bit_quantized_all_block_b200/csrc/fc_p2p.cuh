// fc_p2p.cuh -- the two-step quantized all-reduce across P GPUs as ONE kernel
// per rank (Flash Communication, sciencestack.ai/paper/2412.04964: TL;DR, the
// quantize -> reduce-scatter -> all-gather all-reduce; Fig. 3, one partial per
// tensor-parallel rank).
//
// Rank r's kernel, n elements, chunk c = [c*m, (c+1)*m):
//   phase 1  quantize x_r chunk by chunk into S1_r[c] (rank r's memory), then
//            count this CTA on rank r's phase-1 counter;
//   phase 2  wait until every rank's phase-1 counter reaches epoch * CTAs,
//            then reduce-scatter chunk r: read S1_p[r] from every rank p
//            (peer memory), sum in rank order, requantize into S2_r; count;
//   phase 3  wait for every owner's phase-2 counter, then all-gather: read
//            S2_c from owner c and dequantize into y[chunk c].
// The transfers are the phase-2 and phase-3 loads themselves, so on NVLink
// each tile's movement overlaps the arithmetic on the others.  Counters only
// grow (call k of a sequence waits for k * CTAs), so nothing is reset between
// calls, and the reuse argument of the host-barrier version carries over: a
// rank rewrites S1 only after every owner finished reading it (phase 3 of the
// previous call waited for all phase-2 counts) and S2 only after every rank
// finished reading it (phase 2 waits for all phase-1 counts of the next call).
//
// Visibility: a CTA's payload writes are ordered before its count by a CTA
// barrier and a system-scope fence in the counting thread; a waiting thread
// reads counters with system-scope acquire loads, then releases its CTA with
// a barrier; payloads written during the launch are then read with coherent
// L2 loads (never through the read-only path).  Every wait gives up after 2 s of %globaltimer, ORs 1 into the
// status word and skips the rest of the call, so a missing peer ends the call
// with an error instead of a hang.
//
// The CTAs of all ranks wait on each other, so they must be co-resident: the
// kernel is launched cooperatively.  In the emulated form (EMU) one
// cooperative launch runs all P ranks' CTAs on one GPU, rank = block / CTAs
// per rank, with every rank's buffers in that GPU's memory -- the form in
// which the protocol is tested on a single GPU.
#pragma once

#include "fc_p2p_args.cuh"
#include "fc_staged.cuh"

namespace fc {

constexpr uint64_t P2P_WAIT_NS = 2000000000ull;

__device__ __forceinline__ unsigned int ld_acquire_sys(const unsigned int* p)
{
    unsigned int v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t p2p_now()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Count this CTA's completion of a phase on `ctr` (after its writes).
__device__ __forceinline__ void p2p_count(unsigned int* ctr)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence_system();
        atomicAdd_system(ctr, 1u);
    }
}

// Wait until every one of the P counters reaches `target` (bounded).  Returns
// false, CTA-uniformly, if any wait gave up or another CTA of this rank did.
template <int P>
__device__ __forceinline__ bool p2p_wait(unsigned int* const* ctrs, unsigned int target, int* status,
                                         int* abort_smem)
{
    if (threadIdx.x == 0) {
        int ok = 1;
        const uint64_t t0 = p2p_now();
        for (int p = 0; p < P && ok; p++) {
            while ((int)(ld_acquire_sys(ctrs[p]) - target) < 0) {
                if (p2p_now() - t0 > P2P_WAIT_NS) {
                    ok = 0;
                    atomicOr_system(status, P2P_STATUS_TIMEOUT);
                    break;
                }
                __nanosleep(64);
            }
        }
        *abort_smem = !ok;
    }
    __syncthreads();
    return *abort_smem == 0;
}

// A thread's E codes of a payload written during this launch (by other CTAs
// or other GPUs): coherent loads that bypass L1 and the read-only path, which
// assume data that does not change while the kernel runs.
template <int BITS, int NC>
__device__ __forceinline__ void load_codes_cg(const uint8_t* codes, size_t e, uint32_t* w)
{
    constexpr int NW = NC * BITS / 4;
    const uint8_t* p = codes + e * BITS / 8;
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 4) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p + 4 * i));
            w[i] = v.x;
            w[i + 1] = v.y;
            w[i + 2] = v.z;
            w[i + 3] = v.w;
        }
    } else {
        const uint2 v = __ldcg(reinterpret_cast<const uint2*>(p));
        w[0] = v.x;
        w[1] = v.y;
    }
}

template <class T, int BITS, int P, bool EMU>
__global__ void __launch_bounds__(P2P_THREADS) k_p2p(const __grid_constant__ P2PArgs a)
{
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
    constexpr int NC = P2P_NC, E = P2P_E, TILE = P2P_TILE;
    constexpr int NW = NC * BITS / 4;
    __shared__ uint32_t red16[P2P_THREADS / 32];
    __shared__ float2 red32[P2P_THREADS / 32];
    __shared__ int abort_smem;

    const int rank = EMU ? (int)blockIdx.x / a.cpr : a.rank;
    const int cta = EMU ? (int)blockIdx.x % a.cpr : (int)blockIdx.x;
    const int io = EMU ? rank : 0;
    const T* x = static_cast<const T*>(a.x[io]);
    T* y = static_cast<T*>(a.y[io]);
    const size_t m = a.m, n = (size_t)P * m;
    const int L = a.block / E;
    const int j = threadIdx.x % L;
    const int lg_block = __ffs(a.block) - 1;
    const size_t toff = (size_t)threadIdx.x * E;
    // The epoch: given (the k-th call on the counters passes k), or 0 = derived
    // from this rank's own phase-1 counter.  After k complete calls it holds
    // k * cpr, and before this CTA counts it can have gained at most cpr - 1
    // counts of this call, so floor(read / cpr) + 1 is this call's epoch.  No
    // argument then changes from call to call, so a CUDA graph can replay it.
    const unsigned int cpr = (unsigned int)a.cpr;
    const unsigned int epoch = a.epoch != 0 ? a.epoch : __ldcg(a.ctr1[rank]) / cpr + 1;
    const unsigned int target = epoch * cpr;

    // ---- phase 1: quantize every chunk of my partial into S1_rank[c] ----------
    for (size_t base = (size_t)cta * TILE; base < n; base += (size_t)a.cpr * TILE) {
        const size_t e = base + toff;
        const bool valid = e < n;
        uint4 raw[NC];
        if (valid) {
            load_chunks<T, NC>(raw, x + e);
        } else {
#pragma unroll
            for (int c = 0; c < NC; c++)
                raw[c] = make_uint4(0, 0, 0, 0);
        }
        const T2 t = as_t2<T2>(group_min_negmax<T>(local_min_negmax<T, NC>(raw), L, red16));
        const float mx = fmaxf(-P2::hi(t), 0.0f);
        const BlockQ b = block_q<BITS>(fminf(P2::lo(t), 0.0f), mx);
        const bool clamp = __any_sync(0xffffffffu, top_code_overflows(mx, b));
        if (valid) {
            float v[E];
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
            const size_t ch = e / m, el = e - ch * m;   // a thread's elements lie in one block, one chunk
            if (clamp)
                quant_store<BITS, NC, true>(v, b, a.s1[rank][ch], el, j == 0, el >> lg_block);
            else
                quant_store<BITS, NC, false>(v, b, a.s1[rank][ch], el, j == 0, el >> lg_block);
        }
    }
    p2p_count(a.ctr1[rank]);

    // ---- phase 2: reduce-scatter my chunk, reading every rank's S1 -------------
    if (!p2p_wait<P>(a.ctr1, target, a.status, &abort_smem))
        return;
    for (size_t base = (size_t)cta * TILE; base < m; base += (size_t)a.cpr * TILE) {
        const size_t el = base + toff;
        const bool valid = el < m;
        const size_t k = el >> lg_block;
        float acc[E];
#pragma unroll
        for (int r = 0; r < P; r++) {
            uint32_t w[NW];
            float s = 1.0f, mz = FC_MAGIC;
            if (valid) {
                const QPtr& q = a.s1[r][rank];
                load_codes_cg<BITS, NC>(q.codes, el, w);
                s = __ldcg(q.scales + k);
                mz = __uint_as_float(FC_MAGIC_BITS + __ldcg(q.zps + k));
            } else {
#pragma unroll
                for (int i = 0; i < NW; i++)
                    w[i] = 0;
            }
            const float2 nmz2 = dup2(-mz), s2 = dup2(s);
#pragma unroll
            for (int c = 0; c < NC; c++) {
                float sh[8];
                chunk_shifted<BITS>(w, c, sh);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float2 xh = prod2(add2(ld2(sh, i), nmz2), s2);    // (q - z) * s
                    st2(acc, c * 8 + i, (r == 0) ? xh : add2(ld2(acc, c * 8 + i), xh));
                }
            }
        }
        float mn = fminf(acc[0], 0.0f), mx = fmaxf(acc[0], 0.0f);
#pragma unroll
        for (int i = 1; i + 1 < E; i += 2) {
            mn = min3(mn, acc[i], acc[i + 1]);
            mx = max3(mx, acc[i], acc[i + 1]);
        }
        mn = fminf(mn, acc[E - 1]);
        mx = fmaxf(mx, acc[E - 1]);
        group_minmax_f32<true>(mn, mx, L, red32);
        const BlockQ b = block_q<BITS>(mn, mx);
        const bool clamp = __any_sync(0xffffffffu, top_code_overflows(mx, b));
        if (valid) {
            if (clamp)
                quant_store<BITS, NC, true>(acc, b, a.s2[rank], el, j == 0, k);
            else
                quant_store<BITS, NC, false>(acc, b, a.s2[rank], el, j == 0, k);
        }
    }
    p2p_count(a.ctr2[rank]);

    // ---- phase 3: all-gather every owner's S2 into y ----------------------------
    if (!p2p_wait<P>(a.ctr2, target, a.status, &abort_smem))
        return;
    for (size_t base = (size_t)cta * TILE; base < n; base += (size_t)a.cpr * TILE) {
        const size_t e = base + toff;
        if (e >= n)
            continue;
        const size_t ch = e / m, el = e - ch * m;
        const QPtr& q = a.s2[ch];
        const size_t k = el >> lg_block;
        uint32_t w[NW];
        load_codes_cg<BITS, NC>(q.codes, el, w);
        const float2 s2 = dup2(__ldcg(q.scales + k));
        const float2 nmz2 = dup2(-__uint_as_float(FC_MAGIC_BITS + __ldcg(q.zps + k)));
        uint4 ov[NC];
#pragma unroll
        for (int c = 0; c < NC; c++) {
            float sh[8], v[8];
            chunk_shifted<BITS>(w, c, sh);
#pragma unroll
            for (int i = 0; i < 8; i += 2)
                st2(v, i, mul2(add2(ld2(sh, i), nmz2), s2));   // (q - z) * s, the product rounded alone
            ov[c] = narrow8<T>(v);
        }
        store_chunks<NC, false>(y + e, ov);
    }
}

template <class T, int BITS, int P, bool EMU>
cudaError_t launch_p2p(const P2PArgs& a, int grid, cudaStream_t st)
{
    void* args[] = {const_cast<P2PArgs*>(&a)};
    return cudaLaunchCooperativeKernel((const void*)k_p2p<T, BITS, P, EMU>, dim3(grid), dim3(P2P_THREADS), args, 0,
                                       st);
}

template <class T, int BITS, int P, bool EMU>
cudaError_t p2p_max_ctas(int* ctas)
{
    int sms = 0, per_sm = 0;
    const cudaError_t e = kernel_residency((const void*)k_p2p<T, BITS, P, EMU>, P2P_THREADS, &sms, &per_sm);
    *ctas = sms * per_sm;     // every CTA must be co-resident: no rounding up
    return e;
}

}  // namespace fc
