/*
 * fc.h -- C ABI of the B200 (sm_100a) low-bit two-step quantized all-reduce.
 *
 * The method is Flash Communication ("Flash Communication: Reducing Tensor
 * Parallelization Bottleneck for Fast Large Language Model Inference",
 * sciencestack.ai/paper/2412.04964): tensor-parallel activation partial sums
 * are quantized to a few bits per value before they are exchanged, and the
 * all-reduce runs in two steps, a reduce-scatter followed by an all-gather
 * (TL;DR; Fig. 3; Fig. 5 right).  Quantization is per block of contiguous
 * elements along the hidden dimension (Fig. 4).  This library runs all P
 * ranks of one all-reduce on one GPU: rank r's partial is a buffer in that
 * GPU's memory, and "sending" a chunk to its owner is reading it.
 *
 * Arithmetic (the page gives no formulas; these are the plainest readings).
 * For a block of B values v_i (fp32; fp16/bf16 inputs are widened exactly),
 * at b bits with qmax = 2^b - 1, every operation binary32, round to nearest
 * even; rne(a*b) rounds the exact product to the nearest integer (ties to
 * even) in one step, and no other operation is fused:
 *   mn = min(0, v_i)   mx = max(0, v_i)
 *   s  = (mx == mn) ? 1 : (mx - mn) / qmax      inv = 1 / s
 *   z  = clamp(rne(-mn * inv), 0, qmax)          (uint8 zero-point)
 *   q_i = clamp(rne(v_i * inv) + z, 0, qmax)     (code)
 *   xhat_i = (q_i - z) * s
 * Reduce-scatter: chunk c = elements [c*n/P, (c+1)*n/P) is dequantized from
 * every rank's step-1 payload and summed in fp32 in rank order 0..P-1 (the
 * sum starts from rank 0's value), then requantized with the same rules
 * (step-2 payload).  All-gather: the step-2 payload is dequantized and
 * rounded (nearest even) to fp16/bf16.  Results are bit-identical to the CPU
 * definition shipped with the tests.
 *
 * Payload layout (structure of arrays, one per quantization):
 *   codes  : n*b/8 bytes.  INT8: one code per byte.  INT4: two codes per
 *            byte, element 2j in the low nibble, element 2j+1 in the high.
 *   scales : n/block fp32, scale of block k at index k.
 *   zps    : n/block uint8, zero-point of block k at index k.
 * Block k covers elements [k*block, (k+1)*block) of the flat tensor.
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers must be CUDA device memory (or
 *     managed memory) of the current device, or page-locked host memory
 *     mapped into the device's address space, given by its device address
 *     (fc_host_device_pointer); the kernels then read and write that host
 *     memory over the bus themselves (zero-copy).  Arrays of pointers and the
 *     fc_qbuf structs themselves live in host memory and are read before the
 *     call returns.  The caller owns every buffer; the library allocates
 *     nothing and keeps no reference after the call.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronizing.
 *   - Arguments are validated on the host before anything is launched.
 *     bits must be 4 or 8; block a power of two in [32, 4096]; P in [1, 8];
 *     n a multiple of block (and of P*block where chunks are involved).
 *     n == 0 is a no-op returning FC_OK (pointers are then not inspected).
 *     Every device pointer must be non-NULL and 16-byte aligned.  When the
 *     inputs and the output are also 32-byte aligned, the fused all-reduce
 *     (equal widths) and the all-gather step move them with 32-byte accesses,
 *     which is faster; the results are the same bits either way.
 *     Output buffers must not overlap input buffers or one another (checked
 *     before launch: FC_ERR_INVALID_ARG).
 *   - Inputs must be finite.  For bf16, every block whose range is nonzero
 *     must have a range in [2^-100, 2^100]; outside that the scale or its
 *     reciprocal may not be finite and the results are unspecified (the
 *     kernels still finish and never trap).
 *   - A CUDA launch failure returns FC_ERR_CUDA; fc_last_cuda_error() then
 *     gives the cudaError_t value (per calling thread).
 */
#ifndef FC_H
#define FC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FC_OK = 0,
    FC_ERR_INVALID_ARG = 1, /* bad size, bits, block, P, NULL or overlapping buffers */
    FC_ERR_UNSUPPORTED = 2, /* a combination the library does not provide         */
    FC_ERR_MISALIGNED = 3,  /* a device pointer is not 16-byte aligned             */
    FC_ERR_CUDA = 4,        /* a CUDA call failed; see fc_last_cuda_error()       */
    FC_ERR_TOO_LARGE = 5    /* needs more than the library's fixed scratch memory */
} fc_status;

typedef enum { FC_FP16 = 0, FC_BF16 = 1 } fc_dtype;

/* One quantized payload (device pointers), layout as described above. */
typedef struct {
    uint8_t* codes;
    float* scales;
    uint8_t* zps;
} fc_qbuf;

/* Sizes of one payload for n elements: *code_bytes = n*bits/8 and
 * *n_blocks = n/block (entries of scales and of zps).  Host only.
 * Errors: FC_ERR_INVALID_ARG for bad bits/block, n % block != 0, NULL outputs. */
fc_status fc_payload_sizes(size_t n, int bits, int block, size_t* code_bytes, size_t* n_blocks);

/* Step 1 on one rank (page: TL;DR, activations quantized to low bit widths; Fig. 4,
 * per-block granularity): quantize the n fp16/bf16 values at x (device) into
 * the payload *out (device buffers).  Requires n % block == 0. */
fc_status fc_quantize(const void* x, fc_dtype dtype, size_t n, int bits, int block,
                      const fc_qbuf* out, void* stream);

/* Step 2, reduce-scatter (page: TL;DR, the first of the two all-reduce steps;
 * Fig. 5 right, the quantization before the reduce-scatter): in[0..P-1] are
 * the P ranks' step-1 payloads of n elements
 * each (host array of P structs of device pointers).  For every chunk c, the
 * owner's work is done: dequantize chunk c from all P payloads, sum in fp32 in
 * rank order 0..P-1, requantize.  *out receives the step-2 payload of all n
 * elements (chunk c at its natural offset, so the P owners' outputs form one
 * payload).  Every block of the result depends only on the same block of the
 * P inputs, so any block-aligned range is valid: one owner of a P-GPU
 * all-reduce passes, for its chunk only, the P ranks' step-1 payload pointers
 * offset to that chunk (peer pointers from fc_ipc_open), n = the chunk length.
 * Requires n % block == 0 (n % (P*block) == 0 for P equal chunks). */
fc_status fc_rs_dequant_sum_requant(const fc_qbuf* in, int P, size_t n, int bits, int block,
                                    const fc_qbuf* out, void* stream);

/* Step 3, all-gather (page: Fig. 5 right, the quantization before the
 * all-gather): dequantize the
 * gathered step-2 payload *in (n elements) and round each value to out_dtype
 * into y (device, n elements).  Requires n % block == 0. */
fc_status fc_ag_dequant(const fc_qbuf* in, size_t n, int bits, int block, fc_dtype out_dtype,
                        void* y, void* stream);

/* The fused all-reduce (page: TL;DR, the method runs as one fused CUDA
 * kernel): x is a host array of P device pointers, each to n fp16/bf16
 * values (rank r's partial).  Writes the all-reduced result, rounded to dtype,
 * to y (device, n elements) in one kernel, without materialising the wire
 * payloads.  When step1 is non-NULL it is a host array of P payloads that
 * receive every rank's step-1 payload; when step2 is non-NULL it receives the
 * step-2 payload.  Results are bit-identical to fc_quantize x P, then
 * fc_rs_dequant_sum_requant, then fc_ag_dequant.  Requires n % (P*block) == 0. */
fc_status fc_quantized_allreduce(const void* const* x, int P, fc_dtype dtype, size_t n, int bits,
                                 int block, void* y, const fc_qbuf* step1, const fc_qbuf* step2,
                                 void* stream);

/* The fused all-reduce with a width per step (page: Fig. 5 right compares the
 * quantization error of the reduce-scatter step with that of the all-gather
 * step).  bits_rs and bits_ag
 * are each 4, 8 or 16; 16 means that step exchanges the fp16/bf16 values
 * unquantized:
 *   bits_rs == 16: the reduce-scatter sums the exactly widened inputs;
 *   bits_ag == 16: the all-gather exchanges the fp32 sum rounded (nearest
 *                  even) to dtype, which is then the output.
 * step1 (P payloads of bits_rs) / step2 (one payload of bits_ag) are optional
 * outputs as for fc_quantized_allreduce, and must be NULL for a step of width
 * 16 (else FC_ERR_INVALID_ARG).  Equal quantized widths are provided for every
 * P in [1, 8]; other combinations for P in {2, 4, 8} (FC_ERR_UNSUPPORTED for
 * the rest).  fc_quantized_allreduce(.., bits, ..) is this call with
 * bits_rs == bits_ag == bits.  Requires n % (P*block) == 0. */
fc_status fc_quantized_allreduce_ex(const void* const* x, int P, fc_dtype dtype, size_t n, int bits_rs,
                                    int bits_ag, int block, void* y, const fc_qbuf* step1,
                                    const fc_qbuf* step2, void* stream);

/* One rank's tensor-parallel partial GEMM with the step-1 quantizer fused into
 * its epilogue (page: Fig. 3, the tensor-parallel block whose attention output
 * projection and MLP down projection produce the partial sums; Fig. 5 left,
 * the all-reduce after each of them).
 *   a       device, [M x K] row-major fp16/bf16 (the rank's activations);
 *   w       device, [N x K] row-major fp16/bf16 (the rank's weight slice, in
 *           the usual [out_features x in_features] layout);
 *   partial = a * w^T with fp32 accumulation on the tensor cores, each value
 *           rounded (nearest even) to dtype.  The summation order inside the
 *           tensor cores is the hardware's, so the partial matches an exact
 *           product to within fp32 accumulation error, not bit for bit.
 *   out     when non-NULL: the step-1 payload of the [M x N] partial at
 *           `bits`, blocks of `block` along N -- bit-identical to calling
 *           fc_quantize on the partial;
 *   partial when non-NULL: receives the [M x N] partial itself.
 *   status  device int, required: set to 0 on the stream before the kernel and
 *           OR-ed with 1 if a pipeline wait inside the kernel gave up (the
 *           kernel then stops early instead of hanging; outputs are invalid).
 * At least one of out / partial must be non-NULL.  Requires M % 128 == 0,
 * N % 256 == 0, K % 64 == 0, block in {32, 64, 128, 256} (a block lies in one
 * row of one 256-column output tile), bits in {4, 8}; 16-byte
 * aligned pointers; outputs must not overlap a or w.  Each call runs one
 * persistent kernel (one CTA per SM, 197 KB shared memory, 512 TMEM columns). */
fc_status fc_gemm_quantize(const void* a, const void* w, fc_dtype dtype, int M, int N, int K, int bits, int block,
                           const fc_qbuf* out, void* partial, int* status, void* stream);

/* The device address of page-locked host memory that is mapped into the
 * device's address space (memory from cudaHostAlloc -- every such allocation
 * is mapped under unified addressing -- or registered with the mapped flag).
 * Passing that address to the entry points above lets a kernel stream its
 * inputs from, or its outputs to, host memory directly.  Host only.
 * Errors: FC_ERR_INVALID_ARG for NULL arguments or memory that is not mapped
 * page-locked host memory. */
fc_status fc_host_device_pointer(const void* host, void** device);

/* Peer memory for the P-GPU deployment (one process per GPU; the page's
 * setting, Fig. 1 and Fig. 3: each rank's payloads live in its own GPU and
 * the other ranks read them over NVLink).  A rank exports the device buffers
 * that hold its payloads; every other rank maps them and passes the mapped
 * pointers to fc_rs_dequant_sum_requant / fc_ag_dequant, whose loads then
 * read the peer's memory directly.  These calls map memory and create no
 * buffers; they synchronize nothing.  Memory from the stream-ordered
 * allocator or from virtual-memory-management reservations cannot be
 * exported (FC_ERR_CUDA). */
#define FC_IPC_HANDLE_BYTES 64

/* Export the device allocation that contains ptr: writes its 64-byte CUDA
 * IPC handle to handle (host memory) and ptr's byte offset inside it to
 * *offset.  Errors: FC_ERR_INVALID_ARG for NULL arguments or a pointer that
 * is not device memory of the current context; FC_ERR_CUDA. */
fc_status fc_ipc_export(const void* ptr, void* handle, size_t* offset);

/* Map an allocation exported by another process (not this one) into this
 * process on the current device, enabling peer access if it lives on another
 * GPU; *base receives the mapping (the exporter's ptr is *base + offset).
 * Errors: FC_ERR_INVALID_ARG for NULL arguments; FC_ERR_CUDA. */
fc_status fc_ipc_open(const void* handle, void** base);

/* Unmap a base returned by fc_ipc_open (after all work that reads it has
 * completed).  Errors: FC_ERR_INVALID_ARG for NULL; FC_ERR_CUDA. */
fc_status fc_ipc_close(void* base);

/* The P-GPU all-reduce as ONE kernel per rank (page: TL;DR, the fused
 * quantize -> reduce-scatter -> all-gather all-reduce; Fig. 3, one partial per
 * tensor-parallel rank).  Rank r's kernel quantizes its partial x (n elements)
 * chunk by chunk into its step-1 payloads, counts on its phase-1 counter, waits
 * for every rank's count, reduce-scatters chunk r by reading every rank's
 * step-1 payload of chunk r (peer memory), writes its step-2 payload, counts on
 * its phase-2 counter, waits, and all-gathers every owner's step-2 payload into
 * y -- bit-identical to fc_quantized_allreduce on the P partials.
 *   rank, P     this rank, P in {2, 4, 8};
 *   x, y        this rank's input and output (device, n fp16/bf16 values);
 *   s1          host array of P*P payloads: s1[p*P + c] = rank p's step-1
 *               payload of chunk c (m = n/P elements each), as this process
 *               addresses it (own memory, or a peer mapping from fc_ipc_open);
 *   s2          host array of P payloads: s2[c] = owner c's step-2 payload of
 *               chunk c (m elements);
 *   ctr1, ctr2  host arrays of P device pointers to rank p's phase counters
 *               (uint32, zero before the first call, never reset);
 *   epoch       k on the k-th call on these counters (1, 2, 3, ...): the call
 *               waits for k * (CTAs per rank) counts; or 0: the kernel derives k
 *               from this rank's phase-1 counter (k-1 complete calls leave
 *               (k-1) * CTAs on it).  Pass 0 in a call that a CUDA graph
 *               captures and replays: a replayed explicit epoch is one that
 *               earlier calls' counts already satisfy, so the ranks would race
 *               (wrong outputs, no error and no hang);
 *   status      device int of this rank: set to 0 on the stream, OR-ed with 1
 *               when a wait gave up after 2 s (a missing or failed peer); the
 *               outputs are then invalid and the counters no longer agree;
 *   ctas_per_rank  0 = as many as can be co-resident (the usual), else a cap;
 *               every rank must use the same value.
 * The counters count CTAs, and the number of CTAs per rank follows n (a
 * problem of fewer tiles than fit on the GPU launches one CTA per tile) and
 * ctas_per_rank: every call on one set of counters must use the same n and
 * ctas_per_rank, whatever the epoch form (a changed CTA count breaks the
 * arithmetic of the targets, and the ranks would race).  Use a separate set of
 * counters for each problem size.
 * The kernel is launched cooperatively (its CTAs wait on each other and on the
 * peers'): no other kernel that waits on this rank may share the GPU.  Requires
 * n % (P*block) == 0, 16-byte-aligned payloads, 4-byte-aligned counters.  The
 * buffers the kernel writes or counts on (y, every payload, every counter, the
 * status word) must not overlap one another or x: FC_ERR_INVALID_ARG before
 * launch.  The ranks' calls must use the same n, bits, block and dtype, and
 * the same epoch (or 0 on every rank). */
fc_status fc_p2p_allreduce(int rank, int P, fc_dtype dtype, size_t n, int bits, int block, const void* x, void* y,
                           const fc_qbuf* s1, const fc_qbuf* s2, unsigned int* const* ctr1,
                           unsigned int* const* ctr2, unsigned int epoch, int* status, int ctas_per_rank,
                           void* stream);

/* fc_p2p_allreduce for all P ranks at once on the current GPU: one
 * cooperative launch whose CTAs play every rank (the protocol of the P-GPU
 * kernel, run where one GPU holds every rank's buffers).  x and y are host
 * arrays of P device pointers (rank p's input and output); s1, s2, ctr1, ctr2
 * and status as above (one status word for all ranks). */
fc_status fc_p2p_allreduce_emulated(int P, fc_dtype dtype, size_t n, int bits, int block, const void* const* x,
                                    void* const* y, const fc_qbuf* s1, const fc_qbuf* s2,
                                    unsigned int* const* ctr1, unsigned int* const* ctr2, unsigned int epoch,
                                    int* status, int ctas_per_rank, void* stream);

/* fc_p2p_allreduce_emulated for callers that cannot allocate device memory.
 * The page has no counterpart: this is a convenience of this library.
 *
 * Who needs it: code that must not call cudaMalloc/cudaFree at the point
 * where it runs the all-reduce -- a plugin whose host framework owns all
 * device memory and forbids allocation inside its execute callback, a serving
 * loop that cannot afford the device-wide synchronisation cudaFree implies,
 * or a process whose memory a caching allocator has already reserved.  Such
 * a caller holds its inputs and outputs but has nowhere to put the wire
 * payloads and the phase counters the all-reduce works through.
 *
 * This entry point keeps all of that scratch (every rank's step-1 chunk
 * payloads, every owner's step-2 payload, the 2*P phase counters and a
 * status word) in one array of FC_NOALLOC_SCRATCH_BYTES bytes of static
 * device memory inside the library.  Every GPU on which the library's module
 * is loaded holds that array until the process exits.  The call allocates
 * nothing: it clears the counters and the status word with cudaMemsetAsync
 * on `stream` and runs the same cooperative kernel as
 * fc_p2p_allreduce_emulated (epoch 1 on the cleared counters), so y equals
 * what fc_p2p_allreduce_emulated and fc_quantized_allreduce produce, bit for
 * bit.
 *   P, dtype, n, bits, block, x, y   as for fc_p2p_allreduce_emulated
 *                                    (P in {2, 4, 8}; x and y host arrays of
 *                                    P device pointers; n per rank);
 *   status   device int, or NULL: set to 0 on the stream, OR-ed with 1 if a
 *            wait inside the kernel gave up (outputs then invalid).  With
 *            NULL that flag stays in the scratch array and nothing reports
 *            it: the call still returns FC_OK.  A caller that must detect a
 *            wait that gave up passes a status word.
 * Scratch needed, with m = n/P and R(v) = v rounded up to a multiple of 256:
 *   256 + P*(P+1) * (R(m*bits/8) + R(4*m/block) + R(m/block)) bytes,
 * e.g. 343 KB for P = 4, n = 65536 per rank, INT8, blocks of 128; at most
 * about 3.2 M elements per rank for P = 4 INT8.  Larger problems return
 * FC_ERR_TOO_LARGE before anything is launched.
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address with cudaGetSymbolAddress, which may load the
 * library's module; make that first call before any stream capture.  Later
 * calls reuse the address while the device's CUDA context is the same one (by
 * its unique context id); the first call after the context was destroyed and
 * re-created (cudaDeviceReset) looks the address up again, so it too belongs
 * before any capture.
 * Every call on a device uses the same array and it keeps the previous
 * call's contents: two calls whose work overlaps on the GPU (different
 * streams without ordering between them, or different host threads) race
 * on it and both results are undefined.  Errors: as for
 * fc_p2p_allreduce_emulated, plus FC_ERR_TOO_LARGE. */
#define FC_NOALLOC_SCRATCH_BYTES (16u << 20)
fc_status fc_p2p_allreduce_emulated_noalloc(int P, fc_dtype dtype, size_t n, int bits, int block,
                                            const void* const* x, void* const* y, int* status, void* stream);

/* Static description of a status code. */
const char* fc_status_string(fc_status status);

/* cudaError_t of the last call on this thread that returned FC_ERR_CUDA (0 if none). */
int fc_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* FC_H */
