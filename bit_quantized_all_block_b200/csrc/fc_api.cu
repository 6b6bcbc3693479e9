// fc_api.cu -- the C ABI (include/fc.h): host-side validation and dispatch.
//
// Every entry point validates its arguments completely before it touches the
// GPU, then launches exactly one kernel on the caller's stream and returns
// without synchronizing.  Nothing is allocated.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "../../include/fc.h"
#include "fc_gemm.cuh"
#include "fc_kernels.cuh"
#include "fc_p2p_args.cuh"

namespace {

thread_local int g_last_cuda_error = 0;

fc_status cuda_fail(cudaError_t e)
{
    g_last_cuda_error = (int)e;
    return FC_ERR_CUDA;
}

bool valid_bits(int bits) { return bits == 4 || bits == 8; }

bool valid_block(int block)
{
    return block >= 32 && block <= 4096 && (block & (block - 1)) == 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Byte ranges [p, p+len) for the overlap checks.
struct Range {
    const void* p;
    size_t len;
};

bool overlap(Range a, Range b)
{
    if (a.len == 0 || b.len == 0)
        return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.len && b0 < a0 + a.len;
}

// Checks a payload's pointers; appends its three ranges to `out`.
fc_status check_qbuf(const fc_qbuf* q, size_t n, int bits, int block, Range* out)
{
    if (q == nullptr || q->codes == nullptr || q->scales == nullptr || q->zps == nullptr)
        return FC_ERR_INVALID_ARG;
    if (!aligned16(q->codes) || !aligned16(q->scales) || !aligned16(q->zps))
        return FC_ERR_MISALIGNED;
    const size_t nb = n / (size_t)block;
    out[0] = {q->codes, n * (size_t)bits / 8};
    out[1] = {q->scales, nb * sizeof(float)};
    out[2] = {q->zps, nb};
    return FC_OK;
}

// Whether an output range overlaps another output or an input (inputs may
// overlap each other).  Sort by start and sweep: of two ranges, the one that
// starts later overlaps the other iff it starts before that one ends, so each
// range is checked against the furthest end seen so far among outputs (and,
// for an output, among all ranges).  Up to kMaxRanges non-empty ranges; more
// are refused as if they overlapped (no caller comes near it).
constexpr int kMaxRanges = 512;

bool any_overlap(const Range* outs, int nout, const Range* ins, int nin)
{
    struct Tagged {
        uintptr_t b, e;
        bool out;
    } r[kMaxRanges];
    int k = 0;
    for (int pass = 0; pass < 2; pass++) {
        const Range* src = pass == 0 ? outs : ins;
        const int cnt = pass == 0 ? nout : nin;
        for (int i = 0; i < cnt; i++) {
            if (src[i].len == 0)
                continue;
            if (k == kMaxRanges)
                return true;
            const uintptr_t b = reinterpret_cast<uintptr_t>(src[i].p);
            r[k++] = {b, b + src[i].len, pass == 0};
        }
    }
    std::sort(r, r + k, [](const Tagged& a, const Tagged& b) { return a.b < b.b; });
    uintptr_t end_out = 0, end_any = 0;
    for (int i = 0; i < k; i++) {
        if (r[i].b < (r[i].out ? end_any : end_out))
            return true;
        end_any = r[i].e > end_any ? r[i].e : end_any;
        if (r[i].out)
            end_out = r[i].e > end_out ? r[i].e : end_out;
    }
    return false;
}

fc::QPtr qptr(const fc_qbuf* q)
{
    if (q == nullptr)
        return fc::QPtr{nullptr, nullptr, nullptr};
    return fc::QPtr{q->codes, q->scales, q->zps};
}

using QuantFnT = cudaError_t (*)(const fc::QuantArgs&, cudaStream_t);
using RsFnT = cudaError_t (*)(const fc::RsArgs&, cudaStream_t);
using AgFnT = cudaError_t (*)(const fc::AgArgs&, cudaStream_t);
using FusedFnT = cudaError_t (*)(const fc::FusedArgs&, cudaStream_t);

// [dtype][bits == 4]
const QuantFnT kQuant[2][2] = {
    {fc::launch_quantize<__half, 8>, fc::launch_quantize<__half, 4>},
    {fc::launch_quantize<__nv_bfloat16, 8>, fc::launch_quantize<__nv_bfloat16, 4>},
};
const AgFnT kAg[2][2] = {
    {fc::launch_ag<__half, 8>, fc::launch_ag<__half, 4>},
    {fc::launch_ag<__nv_bfloat16, 8>, fc::launch_ag<__nv_bfloat16, 4>},
};
// The same with 32-byte accesses, for y and codes 32-byte aligned.
const AgFnT kAgWide[2][2] = {
    {fc::launch_ag<__half, 8, true>, fc::launch_ag<__half, 4, true>},
    {fc::launch_ag<__nv_bfloat16, 8, true>, fc::launch_ag<__nv_bfloat16, 4, true>},
};
// [bits == 4][P - 1]
const RsFnT kRs[2][8] = {
    {fc::launch_rs<8, 1>, fc::launch_rs<8, 2>, fc::launch_rs<8, 3>, fc::launch_rs<8, 4>,
     fc::launch_rs<8, 5>, fc::launch_rs<8, 6>, fc::launch_rs<8, 7>, fc::launch_rs<8, 8>},
    {fc::launch_rs<4, 1>, fc::launch_rs<4, 2>, fc::launch_rs<4, 3>, fc::launch_rs<4, 4>,
     fc::launch_rs<4, 5>, fc::launch_rs<4, 6>, fc::launch_rs<4, 7>, fc::launch_rs<4, 8>},
};
// [dtype][width index of the RS step][width index of the AG step][P - 1];
// width index: 4 -> 0, 8 -> 1, 16 -> 2.  Equal quantized widths exist for
// every P; the other combinations for P = 2, 4, 8 (NULL elsewhere).
#define FC_ALLP(T, B1, B2)                                                                        \
    {fc::launch_fused<T, B1, B2, 1>, fc::launch_fused<T, B1, B2, 2>, fc::launch_fused<T, B1, B2, 3>, \
     fc::launch_fused<T, B1, B2, 4>, fc::launch_fused<T, B1, B2, 5>, fc::launch_fused<T, B1, B2, 6>, \
     fc::launch_fused<T, B1, B2, 7>, fc::launch_fused<T, B1, B2, 8>}
#define FC_P248(T, B1, B2)                                                                        \
    {nullptr, fc::launch_fused<T, B1, B2, 2>, nullptr, fc::launch_fused<T, B1, B2, 4>,            \
     nullptr, nullptr, nullptr, fc::launch_fused<T, B1, B2, 8>}
#define FC_DTYPE(T)                                                                               \
    {{FC_ALLP(T, 4, 4), FC_P248(T, 4, 8), FC_P248(T, 4, 16)},                                    \
     {FC_P248(T, 8, 4), FC_ALLP(T, 8, 8), FC_P248(T, 8, 16)},                                    \
     {FC_P248(T, 16, 4), FC_P248(T, 16, 8), FC_P248(T, 16, 16)}}
const FusedFnT kFused[2][3][3][8] = {FC_DTYPE(__half), FC_DTYPE(__nv_bfloat16)};
#undef FC_DTYPE
#undef FC_P248
#undef FC_ALLP
// Equal quantized widths with 32-byte accesses of the inputs and the output,
// for every x[r] and y 32-byte aligned: [dtype][bits == 4][P - 1].
#define FC_WIDE(T, B)                                                                              \
    {fc::launch_fused<T, B, B, 1, false, true>, fc::launch_fused<T, B, B, 2, false, true>,           \
     fc::launch_fused<T, B, B, 3, false, true>, fc::launch_fused<T, B, B, 4, false, true>,           \
     fc::launch_fused<T, B, B, 5, false, true>, fc::launch_fused<T, B, B, 6, false, true>,           \
     fc::launch_fused<T, B, B, 7, false, true>, fc::launch_fused<T, B, B, 8, false, true>}
const FusedFnT kFusedWide[2][2][8] = {
    {FC_WIDE(__half, 8), FC_WIDE(__half, 4)},
    {FC_WIDE(__nv_bfloat16, 8), FC_WIDE(__nv_bfloat16, 4)},
};
#undef FC_WIDE

// The same for blocks whose thread group is narrower than P lanes (every lane
// computes every rank's scale): quantized reduce-scatter step, P >= 3 (below
// that every group is wide enough).  [dtype][w1][w2][P - 1] as kFused.
#define FC_N3(T, B1, B2)                                                                                  \
    {nullptr, nullptr, fc::launch_fused<T, B1, B2, 3, false, false, false>,                                \
     fc::launch_fused<T, B1, B2, 4, false, false, false>, fc::launch_fused<T, B1, B2, 5, false, false, false>, \
     fc::launch_fused<T, B1, B2, 6, false, false, false>, fc::launch_fused<T, B1, B2, 7, false, false, false>, \
     fc::launch_fused<T, B1, B2, 8, false, false, false>}
#define FC_N48(T, B1, B2)                                                                                 \
    {nullptr, nullptr, nullptr, fc::launch_fused<T, B1, B2, 4, false, false, false>,                      \
     nullptr, nullptr, nullptr, fc::launch_fused<T, B1, B2, 8, false, false, false>}
#define FC_NONE {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr}
#define FC_DTYPE(T)                                                                               \
    {{FC_N3(T, 4, 4), FC_N48(T, 4, 8), FC_N48(T, 4, 16)},                                        \
     {FC_N48(T, 8, 4), FC_N3(T, 8, 8), FC_N48(T, 8, 16)},                                        \
     {FC_NONE, FC_NONE, FC_NONE}}
const FusedFnT kFusedNarrow[2][3][3][8] = {FC_DTYPE(__half), FC_DTYPE(__nv_bfloat16)};
#undef FC_DTYPE
#undef FC_NONE
#undef FC_N48
#undef FC_N3

int width_index(int bits) { return bits == 4 ? 0 : bits == 8 ? 1 : bits == 16 ? 2 : -1; }

// The fused kernel's latency shape (64-thread CTAs, 8 elements per thread) for
// decode-sized messages: equal quantized widths, P in {2, 4, 8}, blocks of at
// most 256, and at most FC_SMALL_MAX_ELEMS elements over all ranks.
#ifndef FC_SMALL_MAX_ELEMS
#define FC_SMALL_MAX_ELEMS (1u << 20)
#endif
#define FC_SMALL(T, B) {fc::launch_fused<T, B, B, 2, true>, fc::launch_fused<T, B, B, 4, true>, fc::launch_fused<T, B, B, 8, true>}
// [dtype][bits == 4][P = 2, 4, 8]
const FusedFnT kFusedSmall[2][2][3] = {
    {FC_SMALL(__half, 8), FC_SMALL(__half, 4)},
    {FC_SMALL(__nv_bfloat16, 8), FC_SMALL(__nv_bfloat16, 4)},
};
#undef FC_SMALL

FusedFnT small_variant(fc_dtype dtype, int bits_rs, int bits_ag, int P, int block, size_t n)
{
    if (bits_rs != bits_ag || bits_rs == 16 || block > 256 || n * (size_t)P > (size_t)FC_SMALL_MAX_ELEMS ||
        !fc::fused_lane_split(block, P, true))
        return nullptr;
    const int pi = P == 2 ? 0 : P == 4 ? 1 : P == 8 ? 2 : -1;
    return pi < 0 ? nullptr : kFusedSmall[dtype][bits_rs == 4][pi];
}

}  // namespace

namespace fc {

cudaError_t kernel_residency(const void* kernel, int threads, int* sms, int* per_sm)
{
    static std::mutex mu;
    // (device, kernel, threads) -> (SMs, co-resident CTAs per SM); the queries
    // cost microseconds of host time, more than a decode-sized launch
    static std::map<std::tuple<int, const void*, int>, std::pair<int, int>> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find({dev, kernel, threads});
    if (it == cache.end()) {
        int n_sm = 0, n_cta = 0;
        e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n_cta, kernel, threads, 0);
        if (e != cudaSuccess)
            return e;
        it = cache.emplace(std::make_tuple(dev, kernel, threads), std::make_pair(n_sm, n_cta)).first;
    }
    *sms = it->second.first;
    *per_sm = it->second.second;
    return cudaSuccess;
}

cudaError_t persistent_grid(const void* kernel, int threads, size_t n, size_t tile, int* grid)
{
    int sms = 0, per_sm = 0;
    cudaError_t e = kernel_residency(kernel, threads, &sms, &per_sm);
    if (e != cudaSuccess)
        return e;
    const int ctas = sms * (per_sm > 0 ? per_sm : 1);
    const size_t tiles = (n + tile - 1) / tile;
    *grid = (int)(tiles < (size_t)ctas ? tiles : (size_t)ctas);
    return cudaSuccess;
}

}  // namespace fc

extern "C" {

fc_status fc_payload_sizes(size_t n, int bits, int block, size_t* code_bytes, size_t* n_blocks)
{
    if (!valid_bits(bits) || !valid_block(block) || n % (size_t)block != 0 || code_bytes == nullptr ||
        n_blocks == nullptr)
        return FC_ERR_INVALID_ARG;
    *code_bytes = n * (size_t)bits / 8;
    *n_blocks = n / (size_t)block;
    return FC_OK;
}

fc_status fc_quantize(const void* x, fc_dtype dtype, size_t n, int bits, int block, const fc_qbuf* out,
                      void* stream)
{
    if (!valid_bits(bits) || !valid_block(block) || (dtype != FC_FP16 && dtype != FC_BF16) ||
        n % (size_t)block != 0)
        return FC_ERR_INVALID_ARG;
    if (n == 0)
        return FC_OK;
    if (x == nullptr)
        return FC_ERR_INVALID_ARG;
    if (!aligned16(x))
        return FC_ERR_MISALIGNED;
    Range outs[3];
    fc_status st = check_qbuf(out, n, bits, block, outs);
    if (st != FC_OK)
        return st;
    const Range in{x, n * 2};
    if (any_overlap(outs, 3, &in, 1))
        return FC_ERR_INVALID_ARG;
    fc::QuantArgs a{x, qptr(out), n, block};
    cudaError_t e = kQuant[dtype][bits == 4](a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}

fc_status fc_rs_dequant_sum_requant(const fc_qbuf* in, int P, size_t n, int bits, int block,
                                    const fc_qbuf* out, void* stream)
{
    // Each block of the sum depends only on the same block of every rank, so
    // any whole number of blocks is a valid range (one owner's chunk included).
    if (!valid_bits(bits) || !valid_block(block) || P < 1 || P > fc::FC_MAX_P || n % (size_t)block != 0)
        return FC_ERR_INVALID_ARG;
    if (n == 0)
        return FC_OK;
    if (in == nullptr)
        return FC_ERR_INVALID_ARG;
    Range ins[3 * fc::FC_MAX_P], outs[3];
    for (int r = 0; r < P; r++) {
        fc_status st = check_qbuf(&in[r], n, bits, block, ins + 3 * r);
        if (st != FC_OK)
            return st;
    }
    fc_status st = check_qbuf(out, n, bits, block, outs);
    if (st != FC_OK)
        return st;
    if (any_overlap(outs, 3, ins, 3 * P))
        return FC_ERR_INVALID_ARG;
    fc::RsArgs a{};
    for (int r = 0; r < P; r++)
        a.in[r] = qptr(&in[r]);
    a.out = qptr(out);
    a.n = n;
    a.block = block;
    cudaError_t e = kRs[bits == 4][P - 1](a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}

fc_status fc_ag_dequant(const fc_qbuf* in, size_t n, int bits, int block, fc_dtype out_dtype, void* y,
                        void* stream)
{
    if (!valid_bits(bits) || !valid_block(block) || (out_dtype != FC_FP16 && out_dtype != FC_BF16) ||
        n % (size_t)block != 0)
        return FC_ERR_INVALID_ARG;
    if (n == 0)
        return FC_OK;
    Range ins[3];
    fc_status st = check_qbuf(in, n, bits, block, ins);
    if (st != FC_OK)
        return st;
    if (y == nullptr)
        return FC_ERR_INVALID_ARG;
    if (!aligned16(y))
        return FC_ERR_MISALIGNED;
    const Range out{y, n * 2};
    if (any_overlap(&out, 1, ins, 3))
        return FC_ERR_INVALID_ARG;
    fc::AgArgs a{qptr(in), y, n, block};
    const bool wide = aligned32(y) && aligned32(in->codes);
    cudaError_t e = (wide ? kAgWide : kAg)[out_dtype][bits == 4](a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}

fc_status fc_quantized_allreduce_ex(const void* const* x, int P, fc_dtype dtype, size_t n, int bits_rs,
                                    int bits_ag, int block, void* y, const fc_qbuf* step1,
                                    const fc_qbuf* step2, void* stream)
{
    const int w1 = width_index(bits_rs), w2 = width_index(bits_ag);
    if (w1 < 0 || w2 < 0 || !valid_block(block) || (dtype != FC_FP16 && dtype != FC_BF16) || P < 1 ||
        P > fc::FC_MAX_P || n % ((size_t)P * (size_t)block) != 0)
        return FC_ERR_INVALID_ARG;
    if ((bits_rs == 16 && step1 != nullptr) || (bits_ag == 16 && step2 != nullptr))
        return FC_ERR_INVALID_ARG;   // an unquantized step has no payload
    FusedFnT fn = kFused[dtype][w1][w2][P - 1];
    if (fn == nullptr)
        return FC_ERR_UNSUPPORTED;
    const bool split = w1 == 2 || fc::fused_lane_split(block, P, false);   // no scales when RS is unquantized
    if (!split)
        fn = kFusedNarrow[dtype][w1][w2][P - 1];
    FusedFnT small = small_variant(dtype, bits_rs, bits_ag, P, block, n);
    if (small != nullptr)
        fn = small;
    if (n == 0)
        return FC_OK;
    if (x == nullptr || y == nullptr)
        return FC_ERR_INVALID_ARG;
    Range ins[fc::FC_MAX_P];
    for (int r = 0; r < P; r++) {
        if (x[r] == nullptr)
            return FC_ERR_INVALID_ARG;
        if (!aligned16(x[r]))
            return FC_ERR_MISALIGNED;
        ins[r] = {x[r], n * 2};
    }
    if (!aligned16(y))
        return FC_ERR_MISALIGNED;
    Range outs[1 + 3 * (fc::FC_MAX_P + 1)];
    int nout = 0;
    outs[nout++] = {y, n * 2};
    if (step1 != nullptr) {
        for (int r = 0; r < P; r++) {
            fc_status st = check_qbuf(&step1[r], n, bits_rs, block, outs + nout);
            if (st != FC_OK)
                return st;
            nout += 3;
        }
    }
    if (step2 != nullptr) {
        fc_status st = check_qbuf(step2, n, bits_ag, block, outs + nout);
        if (st != FC_OK)
            return st;
        nout += 3;
    }
    if (any_overlap(outs, nout, ins, P))
        return FC_ERR_INVALID_ARG;
    if (small == nullptr && split && bits_rs == bits_ag && bits_rs != 16) {
        bool wide = aligned32(y);
        for (int r = 0; r < P; r++)
            wide = wide && aligned32(x[r]);
        if (wide)
            fn = kFusedWide[dtype][bits_rs == 4][P - 1];
    }
    fc::FusedArgs a{};
    for (int r = 0; r < P; r++) {
        a.x[r] = x[r];
        a.step1[r] = step1 ? qptr(&step1[r]) : fc::QPtr{nullptr, nullptr, nullptr};
    }
    a.step2 = qptr(step2);
    a.y = y;
    a.n = n;
    a.block = block;
    a.write_step1 = step1 != nullptr;
    a.write_step2 = step2 != nullptr;
    cudaError_t e = fn(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}

fc_status fc_quantized_allreduce(const void* const* x, int P, fc_dtype dtype, size_t n, int bits, int block,
                                 void* y, const fc_qbuf* step1, const fc_qbuf* step2, void* stream)
{
    if (!valid_bits(bits))
        return FC_ERR_INVALID_ARG;
    return fc_quantized_allreduce_ex(x, P, dtype, n, bits, bits, block, y, step1, step2, stream);
}

}  // extern "C"

namespace {

// cuTensorMapEncodeTiled from the driver, fetched once through the runtime
// (no link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
    });
    return fn;
}

// 2-D tensor map of a row-major [rows x K] 16-bit matrix, boxes of
// box_rows x 64 elements (128 bytes along K) with the 128-byte swizzle.
bool make_kmajor_map(CUtensorMap* map, const void* base, bool bf16, uint64_t rows, uint64_t K, uint32_t box_rows)
{
    PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
    if (enc == nullptr)
        return false;
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)fc::GQ_BK, box_rows};
    const cuuint32_t elem[2] = {1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
               const_cast<void*>(base), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using GemmFnT = cudaError_t (*)(const CUtensorMap&, const CUtensorMap&, const fc::GemmQuantArgs&, cudaStream_t);
// [dtype][bits == 4][log2(block) - 5]
#define FC_GEMM_ROW(L, T, B) {L<T, B, 32>, L<T, B, 64>, L<T, B, 128>, L<T, B, 256>}
const GemmFnT kGemm[2][2][4] = {
    {FC_GEMM_ROW(fc::launch_gemm_quant, __half, 8), FC_GEMM_ROW(fc::launch_gemm_quant, __half, 4)},
    {FC_GEMM_ROW(fc::launch_gemm_quant, __nv_bfloat16, 8), FC_GEMM_ROW(fc::launch_gemm_quant, __nv_bfloat16, 4)},
};
// The SM-pair kernel (256 x 256 tiles), used when M is a multiple of 256.
const GemmFnT kGemmPair[2][2][4] = {
    {FC_GEMM_ROW(fc::launch_gemm_quant_pair, __half, 8), FC_GEMM_ROW(fc::launch_gemm_quant_pair, __half, 4)},
    {FC_GEMM_ROW(fc::launch_gemm_quant_pair, __nv_bfloat16, 8),
     FC_GEMM_ROW(fc::launch_gemm_quant_pair, __nv_bfloat16, 4)},
};
#undef FC_GEMM_ROW
#ifndef FC_GEMM_PAIR
#define FC_GEMM_PAIR 1
#endif

}  // namespace

// ---- the one-kernel P-GPU all-reduce -------------------------------------------
namespace {
using P2PLaunch = cudaError_t (*)(const fc::P2PArgs&, int, cudaStream_t);
using P2PCtas = cudaError_t (*)(int*);
#define FC_P2P_ROW(T, B, EMU)                                                                   \
    {fc::launch_p2p<T, B, 2, EMU>, fc::launch_p2p<T, B, 4, EMU>, fc::launch_p2p<T, B, 8, EMU>}
#define FC_P2P_CTAS(T, B, EMU)                                                                  \
    {fc::p2p_max_ctas<T, B, 2, EMU>, fc::p2p_max_ctas<T, B, 4, EMU>, fc::p2p_max_ctas<T, B, 8, EMU>}
// [emulated][dtype][bits == 4][P = 2, 4, 8]
const P2PLaunch kP2P[2][2][2][3] = {
    {{FC_P2P_ROW(__half, 8, false), FC_P2P_ROW(__half, 4, false)},
     {FC_P2P_ROW(__nv_bfloat16, 8, false), FC_P2P_ROW(__nv_bfloat16, 4, false)}},
    {{FC_P2P_ROW(__half, 8, true), FC_P2P_ROW(__half, 4, true)},
     {FC_P2P_ROW(__nv_bfloat16, 8, true), FC_P2P_ROW(__nv_bfloat16, 4, true)}},
};
const P2PCtas kP2PCtas[2][2][2][3] = {
    {{FC_P2P_CTAS(__half, 8, false), FC_P2P_CTAS(__half, 4, false)},
     {FC_P2P_CTAS(__nv_bfloat16, 8, false), FC_P2P_CTAS(__nv_bfloat16, 4, false)}},
    {{FC_P2P_CTAS(__half, 8, true), FC_P2P_CTAS(__half, 4, true)},
     {FC_P2P_CTAS(__nv_bfloat16, 8, true), FC_P2P_CTAS(__nv_bfloat16, 4, true)}},
};
#undef FC_P2P_CTAS
#undef FC_P2P_ROW

fc_status p2p_common(bool emu, int rank, int P, fc_dtype dtype, size_t n, int bits, int block,
                     const void* const* x, void* const* y, const fc_qbuf* s1, const fc_qbuf* s2,
                     unsigned int* const* ctr1, unsigned int* const* ctr2, unsigned int epoch, int* status,
                     int ctas_per_rank, void* stream)
{
    const int pi = P == 2 ? 0 : P == 4 ? 1 : P == 8 ? 2 : -1;
    if (pi < 0 || !valid_bits(bits) || !valid_block(block) || (dtype != FC_FP16 && dtype != FC_BF16) ||
        n % ((size_t)P * (size_t)block) != 0 || (!emu && (rank < 0 || rank >= P)) ||
        ctas_per_rank < 0)
        return FC_ERR_INVALID_ARG;
    if (n == 0)
        return FC_OK;
    if (x == nullptr || y == nullptr || s1 == nullptr || s2 == nullptr || ctr1 == nullptr || ctr2 == nullptr ||
        status == nullptr)
        return FC_ERR_INVALID_ARG;
    const size_t m = n / (size_t)P;
    fc::P2PArgs a{};
    const int nio = emu ? P : 1;
    for (int i = 0; i < nio; i++) {
        if (x[i] == nullptr || y[i] == nullptr)
            return FC_ERR_INVALID_ARG;
        if (!aligned16(x[i]) || !aligned16(y[i]))
            return FC_ERR_MISALIGNED;
        a.x[i] = x[i];
        a.y[i] = y[i];
    }
    // every buffer the kernel writes (outputs, payloads, counters, status)
    // must not overlap another one or an input
    Range outs[fc::FC_MAX_P * (1 + 3 * fc::FC_MAX_P + 3 + 2) + 1], ins[fc::FC_MAX_P];
    int nout = 0;
    for (int i = 0; i < nio; i++) {
        outs[nout++] = {y[i], n * 2};
        ins[i] = {x[i], n * 2};
    }
    for (int p = 0; p < P; p++) {
        for (int c = 0; c < P; c++) {
            fc_status st = check_qbuf(&s1[p * P + c], m, bits, block, outs + nout);
            if (st != FC_OK)
                return st;
            nout += 3;
            a.s1[p][c] = qptr(&s1[p * P + c]);
        }
        fc_status st = check_qbuf(&s2[p], m, bits, block, outs + nout);
        if (st != FC_OK)
            return st;
        nout += 3;
        a.s2[p] = qptr(&s2[p]);
        if (ctr1[p] == nullptr || ctr2[p] == nullptr)
            return FC_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(ctr1[p]) & 3u) || (reinterpret_cast<uintptr_t>(ctr2[p]) & 3u))
            return FC_ERR_MISALIGNED;
        outs[nout++] = {ctr1[p], sizeof(unsigned int)};
        outs[nout++] = {ctr2[p], sizeof(unsigned int)};
        a.ctr1[p] = ctr1[p];
        a.ctr2[p] = ctr2[p];
    }
    if (reinterpret_cast<uintptr_t>(status) & 3u)
        return FC_ERR_MISALIGNED;
    outs[nout++] = {status, sizeof(int)};
    if (any_overlap(outs, nout, ins, nio))
        return FC_ERR_INVALID_ARG;
    a.status = status;
    a.m = m;
    a.block = block;
    a.rank = emu ? 0 : rank;
    a.epoch = epoch;
    // co-resident CTAs: all ranks' CTAs wait on each other
    int max_ctas = 0;
    cudaError_t e = kP2PCtas[emu][dtype][bits == 4][pi](&max_ctas);
    if (e != cudaSuccess)
        return cuda_fail(e);
    const int ranks_here = emu ? P : 1;
    const size_t tiles = (n + (size_t)fc::P2P_TILE - 1) / (size_t)fc::P2P_TILE;
    int cpr = max_ctas / ranks_here;
    if (ctas_per_rank > 0 && ctas_per_rank < cpr)
        cpr = ctas_per_rank;
    if ((size_t)cpr > tiles)
        cpr = (int)tiles;
    if (cpr < 1)
        return FC_ERR_UNSUPPORTED;
    a.cpr = cpr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = cudaMemsetAsync(status, 0, sizeof(int), st);
    if (e == cudaSuccess)
        e = kP2P[emu][dtype][bits == 4][pi](a, cpr * ranks_here, st);
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}
}  // namespace

extern "C" {

fc_status fc_gemm_quantize(const void* a, const void* w, fc_dtype dtype, int M, int N, int K, int bits, int block,
                           const fc_qbuf* out, void* partial, int* status, void* stream)
{
    if ((dtype != FC_FP16 && dtype != FC_BF16) || M <= 0 || N <= 0 || K <= 0 || M % fc::GQ_BM != 0 ||
        N % fc::GQ_BN != 0 || K % fc::GQ_BK != 0 || (block != 32 && block != 64 && block != 128 && block != 256) ||
        (out != nullptr && !valid_bits(bits)))
        return FC_ERR_INVALID_ARG;
    if (a == nullptr || w == nullptr || status == nullptr || (out == nullptr && partial == nullptr))
        return FC_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(w) || !aligned16(status) || (partial != nullptr && !aligned16(partial)))
        return FC_ERR_MISALIGNED;
    const size_t n = (size_t)M * (size_t)N;
    const int qbits = out != nullptr ? bits : 8;
    Range ins[2] = {{a, (size_t)M * (size_t)K * 2}, {w, (size_t)N * (size_t)K * 2}};
    Range outs[5];
    int nout = 0;
    outs[nout++] = {status, sizeof(int)};
    if (partial != nullptr)
        outs[nout++] = {partial, n * 2};
    if (out != nullptr) {
        fc_status st = check_qbuf(out, n, qbits, block, outs + nout);
        if (st != FC_OK)
            return st;
        nout += 3;
    }
    if (any_overlap(outs, nout, ins, 2))
        return FC_ERR_INVALID_ARG;
    const bool pair = FC_GEMM_PAIR && M % 256 == 0;   // SM pairs: each CTA loads 128 rows of W
    CUtensorMap ta, tb;
    if (!make_kmajor_map(&ta, a, dtype == FC_BF16, (uint64_t)M, (uint64_t)K, fc::GQ_BM) ||
        !make_kmajor_map(&tb, w, dtype == FC_BF16, (uint64_t)N, (uint64_t)K, pair ? 128 : fc::GQ_BN))
        return FC_ERR_UNSUPPORTED;
    fc::GemmQuantArgs g{};
    g.out = qptr(out);
    g.partial = partial;
    g.status = status;
    g.M = M;
    g.N = N;
    g.K = K;
    g.block = block;
    g.tiles_m = M / fc::GQ_BM;
    g.tiles_n = N / fc::GQ_BN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
    if (e != cudaSuccess)
        return cuda_fail(e);
    const int bi = block == 32 ? 0 : block == 64 ? 1 : block == 128 ? 2 : 3;
    e = (pair ? kGemmPair : kGemm)[dtype][qbits == 4][bi](ta, tb, g, st);
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}

fc_status fc_host_device_pointer(const void* host, void** device)
{
    if (host == nullptr || device == nullptr)
        return FC_ERR_INVALID_ARG;
    void* d = nullptr;
    cudaError_t e = cudaHostGetDevicePointer(&d, const_cast<void*>(host), 0);
    if (e != cudaSuccess || d == nullptr) {
        cudaGetLastError();   // not mapped page-locked memory; keep the error out of later launch checks
        return FC_ERR_INVALID_ARG;
    }
    *device = d;
    return FC_OK;
}


// ---- the one-kernel P-GPU all-reduce (entry points) ---------------------------
fc_status fc_p2p_allreduce(int rank, int P, fc_dtype dtype, size_t n, int bits, int block, const void* x, void* y,
                           const fc_qbuf* s1, const fc_qbuf* s2, unsigned int* const* ctr1,
                           unsigned int* const* ctr2, unsigned int epoch, int* status, int ctas_per_rank,
                           void* stream)
{
    return p2p_common(false, rank, P, dtype, n, bits, block, &x, &y, s1, s2, ctr1, ctr2, epoch, status,
                      ctas_per_rank, stream);
}

fc_status fc_p2p_allreduce_emulated(int P, fc_dtype dtype, size_t n, int bits, int block, const void* const* x,
                                    void* const* y, const fc_qbuf* s1, const fc_qbuf* s2,
                                    unsigned int* const* ctr1, unsigned int* const* ctr2, unsigned int epoch,
                                    int* status, int ctas_per_rank, void* stream)
{
    return p2p_common(true, 0, P, dtype, n, bits, block, x, y, s1, s2, ctr1, ctr2, epoch, status, ctas_per_rank,
                      stream);
}

// ---- peer memory (CUDA IPC) for the P-GPU deployment -------------------------
static_assert(sizeof(cudaIpcMemHandle_t) == FC_IPC_HANDLE_BYTES, "IPC handle size");

fc_status fc_ipc_export(const void* ptr, void* handle, size_t* offset)
{
    if (ptr == nullptr || handle == nullptr || offset == nullptr)
        return FC_ERR_INVALID_ARG;
    static PFN_cuMemGetAddressRange range = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            range = reinterpret_cast<PFN_cuMemGetAddressRange>(p);
    });
    if (range == nullptr)
        return cuda_fail(cudaErrorNotSupported);
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return FC_ERR_INVALID_ARG;   // not device memory of the current context
    cudaIpcMemHandle_t h;
    cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
    if (e != cudaSuccess)
        return cuda_fail(e);
    memcpy(handle, &h, sizeof(h));
    *offset = reinterpret_cast<uintptr_t>(ptr) - static_cast<uintptr_t>(base);
    return FC_OK;
}

fc_status fc_ipc_open(const void* handle, void** base)
{
    if (handle == nullptr || base == nullptr)
        return FC_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof(h));
    cudaError_t e = cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess);
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}

fc_status fc_ipc_close(void* base)
{
    if (base == nullptr)
        return FC_ERR_INVALID_ARG;
    cudaError_t e = cudaIpcCloseMemHandle(base);
    return e == cudaSuccess ? FC_OK : cuda_fail(e);
}

const char* fc_status_string(fc_status status)
{
    switch (status) {
    case FC_OK: return "ok";
    case FC_ERR_INVALID_ARG: return "invalid argument (size, bits, block, P, NULL or overlapping buffer)";
    case FC_ERR_UNSUPPORTED: return "unsupported combination";
    case FC_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case FC_ERR_CUDA: return "CUDA error (see fc_last_cuda_error)";
    case FC_ERR_TOO_LARGE: return "problem needs more than the library's fixed scratch memory";
    }
    return "unknown status";
}

int fc_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"

// ---- the all-reduce for callers that cannot allocate device memory ------------
// fc_p2p_allreduce_emulated with its scratch (step-1 and step-2 payloads, phase
// counters, status word) in a fixed array of static device memory instead of
// caller buffers.  Layout, every piece 256-byte aligned:
//   [0, 256)  ctr1[0..P) at words 0..7, ctr2[0..P) at words 8..15, status at 16
//   then s1[p][c] for p, c in [0, P) and s2[c] for c in [0, P), each
//   codes R(m*bits/8), scales R(4*m/block), zps R(m/block).
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FC_NOALLOC_SCRATCH_BYTES];

constexpr size_t kNoallocHeader = 256;
constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
unsigned char* g_noalloc_addr[kNoallocMaxDevices];        // device address of the array, per device
unsigned long long g_noalloc_ctx[kNoallocMaxDevices];     // id of the context that address belongs to

size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

// Unique id of the current CUDA context (ids are never reused within a
// process, so a context created after a reset of the device has a new one);
// false when no context is current or the driver lacks the query.
bool current_context_id(unsigned long long* id)
{
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext ctx = nullptr;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
        return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device: looked up with
// cudaGetSymbolAddress once per device, and again whenever the device's
// context is not the one the address was looked up in (after a reset of the
// device the module, and with it the array, can be loaded at a new address).
fc_status noalloc_scratch(unsigned char** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (dev < 0 || dev >= kNoallocMaxDevices)
        return FC_ERR_UNSUPPORTED;
    unsigned long long ctx = 0;
    const bool known = current_context_id(&ctx);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr || !known || g_noalloc_ctx[dev] != ctx) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess)
            return cuda_fail(e);
        // the lookup may have created the context: take its id now
        g_noalloc_addr[dev] = static_cast<unsigned char*>(ptr);
        g_noalloc_ctx[dev] = current_context_id(&ctx) ? ctx : 0;
    }
    *out = g_noalloc_addr[dev];
    return FC_OK;
}

}  // namespace

extern "C" fc_status fc_p2p_allreduce_emulated_noalloc(int P, fc_dtype dtype, size_t n, int bits, int block,
                                                       const void* const* x, void* const* y, int* status,
                                                       void* stream)
{
    if ((P != 2 && P != 4 && P != 8) || !valid_bits(bits) || !valid_block(block) ||
        (dtype != FC_FP16 && dtype != FC_BF16) || n % ((size_t)P * (size_t)block) != 0)
        return FC_ERR_INVALID_ARG;
    if (n == 0)
        return FC_OK;
    if (x == nullptr || y == nullptr)
        return FC_ERR_INVALID_ARG;
    // the step-1 codes alone take n*bits/8 >= n/2 bytes: this bound keeps the sums below exact
    if (n / 2 > (size_t)FC_NOALLOC_SCRATCH_BYTES)
        return FC_ERR_TOO_LARGE;
    const size_t m = n / (size_t)P;
    const size_t codes = round256(m * (size_t)bits / 8), scales = round256(4 * (m / (size_t)block)),
                 zps = round256(m / (size_t)block);
    const size_t piece = codes + scales + zps;
    if (kNoallocHeader + (size_t)P * (size_t)(P + 1) * piece > (size_t)FC_NOALLOC_SCRATCH_BYTES)
        return FC_ERR_TOO_LARGE;
    unsigned char* base = nullptr;
    fc_status st = noalloc_scratch(&base);
    if (st != FC_OK)
        return st;
    fc_qbuf s1[fc::FC_MAX_P * fc::FC_MAX_P], s2[fc::FC_MAX_P];
    unsigned int* ctr1[fc::FC_MAX_P];
    unsigned int* ctr2[fc::FC_MAX_P];
    unsigned int* words = reinterpret_cast<unsigned int*>(base);
    unsigned char* cur = base + kNoallocHeader;
    auto carve = [&](fc_qbuf* q) {
        q->codes = cur;
        q->scales = reinterpret_cast<float*>(cur + codes);
        q->zps = cur + codes + scales;
        cur += piece;
    };
    for (int i = 0; i < P * P; i++)
        carve(&s1[i]);
    for (int c = 0; c < P; c++) {
        carve(&s2[c]);
        ctr1[c] = words + c;
        ctr2[c] = words + 8 + c;
    }
    int* own_status = reinterpret_cast<int*>(words + 16);
    // counters and the status word start at zero on every call (epoch 1)
    cudaError_t e = cudaMemsetAsync(base, 0, kNoallocHeader, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e);
    return p2p_common(true, 0, P, dtype, n, bits, block, x, y, s1, s2, ctr1, ctr2, 1u,
                      status != nullptr ? status : own_status, 0, stream);
}
