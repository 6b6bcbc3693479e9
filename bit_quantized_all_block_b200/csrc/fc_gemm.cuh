// fc_gemm.cuh -- tensor-parallel partial GEMM with the step-1 quantizer fused
// into its epilogue (sm_100a: TMA -> shared memory -> tcgen05.mma -> TMEM).
//
// Flash Communication (sciencestack.ai/paper/2412.04964) applies its
// quantized all-reduce to the partial sums of the attention output projection
// and of the MLP down projection (Fig. 3: the tensor-parallel LLaMA block;
// Fig. 5 left: the all-reduce after o_proj and after d_proj).  Each rank
// computes partial_r = A_r * W_r^T over its slice of the contraction
// dimension.  Here that GEMM's epilogue rounds the fp32 accumulator to the
// 16-bit partial (exactly what an unfused GEMM would write) and quantizes it
// block by block into the step-1 payload, so the partial never has to be
// written to and re-read from HBM before the reduce-scatter.
//
// Kernel structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0     one lane issues TMA loads of 128x64 A and 256x64 W tiles
//              (128-byte swizzle) into a 4-stage shared-memory ring;
//   warp 1     allocates 512 TMEM columns (two 128x256 fp32 accumulators) and
//              one lane issues tcgen05.mma (M=128, N=256, K=16, bf16/fp16 in,
//              fp32 accumulate), committing each stage back to the producer
//              and each finished accumulator to the epilogue;
//   warps 2-5  the epilogue: each thread owns one row of the tile (its TMEM
//              lane), reads 256 columns with tcgen05.ld, rounds them to the
//              16-bit partial and quantizes its row's blocks in registers --
//              a whole quantization block lives in one thread, so no
//              shuffles are needed -- while the MMA already fills the other
//              accumulator.
// Every mbarrier wait is bounded: after 2 s without progress (timed with
// %globaltimer) the waiting warp raises a CTA-wide abort flag, every other
// wait sees it and stops, in-flight copies and MMAs are drained (again with
// time-bounded waits), TMEM is released and the kernel reports a nonzero
// status word instead of hanging.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "fc_staged.cuh"

namespace fc {

constexpr int GQ_BM = 128, GQ_BN = 256, GQ_BK = 64, GQ_STAGES = 4;
constexpr int GQ_THREADS = 192;
constexpr int GQ_A_BYTES = GQ_BM * GQ_BK * 2;            // 16 KB
constexpr int GQ_B_BYTES = GQ_BN * GQ_BK * 2;            // 32 KB
constexpr int GQ_STAGE_BYTES = GQ_A_BYTES + GQ_B_BYTES;
constexpr int GQ_TMEM_COLS = 2 * GQ_BN;                  // two fp32 accumulators
constexpr int GQ_SMEM_BYTES = GQ_STAGES * GQ_STAGE_BYTES + 1024 /* alignment */ + 256 /* barriers */;
constexpr uint64_t GQ_WAIT_NS = 2000000000ull;          // 2 s: far beyond any legitimate wait

// Status bits reported through the caller's status word.
constexpr int GQ_STATUS_TIMEOUT = 1;

struct GemmQuantArgs {
    QPtr out;          // step-1 payload of the [M x N] partial, or all-null
    void* partial;     // optional [M x N] 16-bit partial (row-major), or nullptr
    int* status;       // device word, OR-ed with GQ_STATUS_* on failure
    int M, N, K;
    int block;
    int tiles_m, tiles_n;
};

// ---- PTX wrappers -----------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity.  Returns false if the
// CTA has aborted, or if GQ_WAIT_NS passed without progress -- then this
// waiter raises the abort flag.  Every legitimate wait in this kernel ends
// within microseconds.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag)
{
    if (mbar_test_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_test_wait(bar, parity))
            return true;
        if ((i & 255u) == 0) {
            if (*abort_flag)
                return false;
            if (global_ns() - t0 > GQ_WAIT_NS) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Drain wait (after an abort): the same time limit, no abort check.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity)
{
    const uint64_t t0 = global_ns();
    while (!mbar_test_wait(bar, parity) && global_ns() - t0 < GQ_WAIT_NS) {
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// Shared-memory matrix descriptor of a K-major tile with 128-byte rows and the
// 128-byte swizzle that the TMA writes: 8-row core groups 1024 bytes apart
// (stride byte offset), leading offset unused (1), descriptor version 1,
// layout type 2 = 128-byte swizzle.  Field layout as in the PTX ISA's
// tcgen05 shared memory descriptor.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(const void* tile)
{
    const uint64_t addr = smem_u32(tile);
    return ((addr & 0x3FFFFull) >> 4) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B both fp16 or
// both bf16, both K-major, M = 128, N = 256.
template <class T>
__host__ __device__ constexpr uint32_t umma_idesc_128x256()
{
    constexpr uint32_t ab = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    return (1u << 4) | (ab << 7) | (ab << 10) | ((uint32_t)(GQ_BN >> 3) << 17) | ((uint32_t)(GQ_BM >> 4) << 24);
}

__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t* r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Tile order: groups of GQ_GROUP_M row blocks, all column blocks of a group
// before the next group, row blocks fastest inside a group.  The tiles that
// run at the same time then share a few row blocks of A and column blocks of
// W, so both stay in L2 even when the operands together exceed it.
constexpr int GQ_GROUP_M = 8;

__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int& m, int& n)
{
    const int per_group = GQ_GROUP_M * tiles_n;
    const int g = tile / per_group;
    const int first_m = g * GQ_GROUP_M;
    const int gsize = min(GQ_GROUP_M, tiles_m - first_m);
    const int r = tile - g * per_group;
    m = first_m + r % gsize;
    n = r / gsize;
}

// ---- epilogue: one row's block of `NB` columns ---------------------------------
// Blocks of more than 128 columns (256: the tile's whole row) would hold 128
// registers of packed values, so they take two passes over TMEM instead, 32
// columns at a time: the first finds the block's extremes of the rounded
// partial (and writes the partial), the second reads the accumulator again,
// rounds it the same way and quantizes.  TMEM reads are cheap next to the
// main loop this epilogue overlaps.
template <class T, int BITS, int NB>
__device__ __forceinline__ void epilogue_block_two_pass(uint32_t taddr, const GemmQuantArgs& a, size_t row, int col)
{
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
    const size_t e = row * (size_t)a.N + col;     // flat element index of the block
    T2 m = P2::from_f2(make_float2(INFINITY, INFINITY)), M = P2::from_f2(make_float2(-INFINITY, -INFINITY));
#pragma unroll 1
    for (int c = 0; c < NB; c += 32) {
        uint32_t r[32], v16[16];
        tmem_ld_32cols(taddr + c, r);
#pragma unroll
        for (int i = 0; i < 16; i++) {
            v16[i] = t2_bits(P2::from_f2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]))));
            m = __hmin2(m, as_t2<T2>(v16[i]));
            M = __hmax2(M, as_t2<T2>(v16[i]));
        }
        if (a.partial != nullptr) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(a.partial) + e + c);
#pragma unroll
            for (int i = 0; i < 4; i++)
                st_stream(dst + i, make_uint4(v16[4 * i], v16[4 * i + 1], v16[4 * i + 2], v16[4 * i + 3]));
        }
    }
    if (a.out.codes == nullptr)
        return;
    const float mn = fminf(fminf(P2::lo(m), P2::hi(m)), 0.0f);
    const float mx = fmaxf(fmaxf(P2::lo(M), P2::hi(M)), 0.0f);
    const BlockQ b = block_q<BITS>(mn, mx);
    const float cqz = __fsub_rn(b.cq, b.zf);
    const uint32_t offset = pack_offset<BITS>(b);
#pragma unroll 1
    for (int c = 0; c < NB; c += 32) {
        uint32_t r[32];
        tmem_ld_32cols(taddr + c, r);
        uint32_t words[BITS];                     // 32 codes: 8 words at INT8, 4 at INT4
#pragma unroll
        for (int g = 0; g < 4; g++) {
            float q[8];
#pragma unroll
            for (int h = 0; h < 4; h++) {
                const float2 f = P2::to_f2(P2::from_f2(make_float2(__uint_as_float(r[8 * g + 2 * h]),
                                                                   __uint_as_float(r[8 * g + 2 * h + 1]))));
                q[2 * h] = fminf(round_product_shifted(f.x, b.inv), cqz);
                q[2 * h + 1] = fminf(round_product_shifted(f.y, b.inv), cqz);
            }
            pack_shifted<BITS>(q, b, offset, words, g);
        }
        uint4* cdst = reinterpret_cast<uint4*>(a.out.codes + (e + c) * BITS / 8);
#pragma unroll
        for (int i = 0; i < BITS / 4; i++)
            st_stream(cdst + i, make_uint4(words[4 * i], words[4 * i + 1], words[4 * i + 2], words[4 * i + 3]));
    }
    const size_t k = e / NB;
    a.out.scales[k] = b.s;
    a.out.zps[k] = zp_byte(b);
}

// Blocks of up to 128 columns: the 16-bit partial values of the block
// (rounded from fp32, nearest even) are kept as packed pairs; the block is
// quantized exactly as fc_quantize would quantize the written partial.
template <class T, int BITS, int NB>
__device__ __forceinline__ void epilogue_block(uint32_t taddr, const GemmQuantArgs& a, size_t row, int col)
{
    if constexpr (NB > 128) {
        epilogue_block_two_pass<T, BITS, NB>(taddr, a, row, col);
        return;
    }
    using P2 = Pair<T>;
    using T2 = typename P2::T2;
    uint32_t v16[NB / 2];
#pragma unroll
    for (int c = 0; c < NB; c += 32) {
        uint32_t r[32];
        tmem_ld_32cols(taddr + c, r);
#pragma unroll
        for (int i = 0; i < 16; i++)
            v16[c / 2 + i] = t2_bits(P2::from_f2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]))));
    }
    if (a.partial != nullptr) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(a.partial) + row * (size_t)a.N + col);
#pragma unroll
        for (int i = 0; i < NB / 8; i++)
            st_stream(dst + i, make_uint4(v16[4 * i], v16[4 * i + 1], v16[4 * i + 2], v16[4 * i + 3]));
    }
    if (a.out.codes == nullptr)
        return;
    T2 m = as_t2<T2>(v16[0]), M = m;
#pragma unroll
    for (int i = 1; i < NB / 2; i++) {
        m = __hmin2(m, as_t2<T2>(v16[i]));
        M = __hmax2(M, as_t2<T2>(v16[i]));
    }
    const float mn = fminf(fminf(P2::lo(m), P2::hi(m)), 0.0f);
    const float mx = fmaxf(fmaxf(P2::lo(M), P2::hi(M)), 0.0f);
    const BlockQ b = block_q<BITS>(mn, mx);
    const float cqz = __fsub_rn(b.cq, b.zf);
    const uint32_t offset = pack_offset<BITS>(b);
    uint32_t words[NB * BITS / 32];
#pragma unroll
    for (int c = 0; c < NB / 8; c++) {
        float r[8];
#pragma unroll
        for (int h = 0; h < 4; h++) {
            const float2 f = P2::to_f2(as_t2<T2>(v16[c * 4 + h]));
            r[2 * h] = fminf(round_product_shifted(f.x, b.inv), cqz);
            r[2 * h + 1] = fminf(round_product_shifted(f.y, b.inv), cqz);
        }
        pack_shifted<BITS>(r, b, offset, words, c);
    }
    const size_t e = row * (size_t)a.N + col;     // flat element index of the block
    uint4* cdst = reinterpret_cast<uint4*>(a.out.codes + e * BITS / 8);
#pragma unroll
    for (int i = 0; i < NB * BITS / 128; i++)
        st_stream(cdst + i, make_uint4(words[4 * i], words[4 * i + 1], words[4 * i + 2], words[4 * i + 3]));
    const size_t k = e / NB;
    a.out.scales[k] = b.s;
    a.out.zps[k] = zp_byte(b);
}

template <class T, int BITS, int NB>
__global__ void __launch_bounds__(GQ_THREADS, 1)
    k_gemm_quant(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const GemmQuantArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + GQ_STAGES * GQ_A_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + GQ_STAGES * GQ_B_BYTES);
    uint64_t* empty = full + GQ_STAGES;
    uint64_t* acc_full = empty + GQ_STAGES;      // [2]
    uint64_t* acc_empty = acc_full + 2;          // [2]
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < GQ_STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);     // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(GQ_TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int num_tiles = a.tiles_m * a.tiles_n;
    const int kblocks = a.K / GQ_BK;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer ----
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0;            // bit s: stage s holds a load not yet seen complete
            uint32_t issued_parity = 0;     // bit s: parity of that load's phase
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                int m_blk, n_blk;
                tile_coords(tile, a.tiles_m, a.tiles_n, m_blk, n_blk);
                for (int kb = 0; kb < kblocks; kb++) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&full[stage], GQ_STAGE_BYTES);
                    tma_load_2d(sA + stage * GQ_A_BYTES, &tmap_a, &full[stage], kb * GQ_BK, m_blk * GQ_BM);
                    tma_load_2d(sB + stage * GQ_B_BYTES, &tmap_b, &full[stage], kb * GQ_BK, n_blk * GQ_BN);
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == GQ_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {   // let every load already issued land before the CTA exits
                for (int s = 0; s < GQ_STAGES; s++) {
                    if (issued & (1u << s))
                        wait_drain(&full[s], (issued_parity >> s) & 1u);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer ----
            constexpr uint32_t idesc = umma_idesc_128x256<T>();
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, any = false;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!wait_bounded(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GQ_BN);
                for (int kb = 0; kb < kblocks; kb++) {
                    if (!wait_bounded(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_k_sw128(sA + stage * GQ_A_BYTES);
                    const uint64_t bd = smem_desc_k_sw128(sB + stage * GQ_B_BYTES);
#pragma unroll
                    for (int k = 0; k < GQ_BK / 16; k++)   // K = 16 per MMA: 32 bytes along the swizzled row
                        umma_f16(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
                    any = true;
                    umma_commit(&empty[stage]);
                    if (++stage == GQ_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                umma_commit(&acc_full[acc]);
                acc ^= 1;
                if (acc == 0)
                    acc_phase ^= 1u;
            }
            if (!ok && any) {   // wait for every MMA already issued before TMEM is freed
                umma_commit(drain);
                wait_drain(drain, 0);
            }
        }
    } else {
        // ---- epilogue: warps 2..5, one TMEM lane quadrant each ----
        const int quad = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            int m_blk, n_blk;
            tile_coords(tile, a.tiles_m, a.tiles_n, m_blk, n_blk);
            if (!wait_bounded(&acc_full[acc], acc_phase, abort_flag))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * GQ_BN);
            const size_t row = (size_t)m_blk * GQ_BM + 32 * quad + lane;
#pragma unroll 1
            for (int c = 0; c < GQ_BN; c += NB)
                epilogue_block<T, BITS, NB>(taddr + c, a, row, n_blk * GQ_BN + c);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[acc]);
            acc ^= 1;
            if (acc == 0)
                acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(GQ_TMEM_COLS)
                     : "memory");
    }
    if (threadIdx.x == 0 && *abort_flag)
        atomicOr(a.status, GQ_STATUS_TIMEOUT);
}

template <class T, int BITS, int NB>
cudaError_t launch_gemm_quant(const CUtensorMap& ta, const CUtensorMap& tb, const GemmQuantArgs& a,
                              cudaStream_t st);


// ============================================================================
// The same GEMM on SM pairs: a cluster of two CTAs computes a 256 x 256 tile
// with tcgen05.mma.cta_group::2 (M = 256 across the pair, N = 256).  Each CTA
// loads its own 128-row halves of the A tile and of the W tile, so each SM
// reads half the W traffic of the one-SM kernel from L2 and a stage is 32 KB,
// which leaves room for 6 stages.  The leader CTA (cluster rank 0) issues the
// MMAs; the loads of both CTAs complete on the leader's stage barrier, the
// leader's commits are multicast to the matching barriers of both CTAs, and
// the epilogue warps of both CTAs arrive on the leader's accumulator barrier.
// Loads carry no multicast: every CTA fetches its own operands.
// ============================================================================
constexpr int G2_STAGES = 6;
constexpr int G2_A_BYTES = 128 * GQ_BK * 2;     // 16 KB: this CTA's 128 rows of A
constexpr int G2_B_BYTES = 128 * GQ_BK * 2;     // 16 KB: this CTA's 128 rows of W (half of N)
constexpr int G2_STAGE_BYTES = G2_A_BYTES + G2_B_BYTES;
constexpr int G2_SMEM_BYTES = G2_STAGES * G2_STAGE_BYTES + 1024 + 256;

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on the barrier at the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint64_t* bar, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on the
// pair leader's barrier (the barrier at the same offset in CTA rank 0, as a
// shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y)
{
    uint32_t leader_bar;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(leader_bar) : "r"(smem_u32(bar)));
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(leader_bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Commit: arrive on the barrier at this offset in both CTAs of the pair once
// every MMA issued so far has completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(smem_u32(bar)), "h"((uint16_t)0x3) : "memory");
}

template <class T>
__host__ __device__ constexpr uint32_t umma_idesc_256x256()
{
    constexpr uint32_t ab = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    return (1u << 4) | (ab << 7) | (ab << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

template <class T, int BITS, int NB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GQ_THREADS, 1)
    k_gemm_quant_pair(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const GemmQuantArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + G2_STAGES * G2_A_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + G2_STAGES * G2_B_BYTES);
    uint64_t* empty = full + G2_STAGES;
    uint64_t* acc_full = empty + G2_STAGES;      // [2]
    uint64_t* acc_empty = acc_full + 2;          // [2] (the leader's is used)
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_rank();
    const bool leader = crank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < G2_STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);     // four epilogue warps in each CTA of the pair
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(GQ_TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();          // both CTAs' barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int tiles_m2 = a.tiles_m / 2;          // 256-row tiles
    const int num_tiles = tiles_m2 * a.tiles_n;
    const int kblocks = a.K / GQ_BK;
    const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer (both CTAs) ----
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_parity = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += num_clusters) {
                int m2, n_blk;
                tile_coords(tile, tiles_m2, a.tiles_n, m2, n_blk);
                const int a_row = m2 * 256 + 128 * (int)crank, b_row = n_blk * GQ_BN + 128 * (int)crank;
                for (int kb = 0; kb < kblocks; kb++) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (leader)
                        mbar_expect_tx(&full[stage], 2 * G2_STAGE_BYTES);
                    tma_load_2d_pair(sA + stage * G2_A_BYTES, &tmap_a, &full[stage], kb * GQ_BK, a_row);
                    tma_load_2d_pair(sB + stage * G2_B_BYTES, &tmap_b, &full[stage], kb * GQ_BK, b_row);
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == G2_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && leader) {   // the leader's stage barriers count both CTAs' loads
                for (int s = 0; s < G2_STAGES; s++)
                    if (issued & (1u << s))
                        wait_drain(&full[s], (issued_parity >> s) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---- MMA issuer (leader CTA) ----
            constexpr uint32_t idesc = umma_idesc_256x256<T>();
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, any = false;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += num_clusters) {
                if (!wait_bounded(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GQ_BN);
                for (int kb = 0; kb < kblocks; kb++) {
                    if (!wait_bounded(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_k_sw128(sA + stage * G2_A_BYTES);
                    const uint64_t bd = smem_desc_k_sw128(sB + stage * G2_B_BYTES);
#pragma unroll
                    for (int k = 0; k < GQ_BK / 16; k++)
                        umma_f16_pair(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
                    any = true;
                    umma_commit_pair(&empty[stage]);
                    if (++stage == G2_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                umma_commit_pair(&acc_full[acc]);
                acc ^= 1;
                if (acc == 0)
                    acc_phase ^= 1u;
            }
            if (!ok && any) {
                umma_commit_pair(drain);
                wait_drain(drain, 0);
            }
        }
    } else {
        // ---- epilogue: warps 2..5 of both CTAs ----
        const int quad = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += num_clusters) {
            int m2, n_blk;
            tile_coords(tile, tiles_m2, a.tiles_n, m2, n_blk);
            if (!wait_bounded(&acc_full[acc], acc_phase, abort_flag))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * GQ_BN);
            const size_t row = (size_t)m2 * 256 + 128 * crank + 32 * quad + lane;
#pragma unroll 1
            for (int c = 0; c < GQ_BN; c += NB)
                epilogue_block<T, BITS, NB>(taddr + c, a, row, n_blk * GQ_BN + c);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(&acc_empty[acc], 0);
            acc ^= 1;
            if (acc == 0)
                acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // neither CTA leaves while the pair's MMAs or barriers are in use
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(GQ_TMEM_COLS)
                     : "memory");
    }
    if (threadIdx.x == 0 && *abort_flag)
        atomicOr(a.status, GQ_STATUS_TIMEOUT);
}

template <class T, int BITS, int NB>
cudaError_t launch_gemm_quant_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmQuantArgs& a,
                                   cudaStream_t st);

}  // namespace fc
