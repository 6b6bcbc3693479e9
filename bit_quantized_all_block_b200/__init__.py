"""B200-native low-bit two-step quantized all-reduce (Flash Communication).

Thin Python binding of the C ABI declared in ``include/fc.h`` (the library is
``libfc.so`` next to this file, built by ``python -m
bit_quantized_all_block_b200.build``).  The functions here carry the C names
and only marshal arguments: torch CUDA tensors supply device pointers, the
current torch stream is passed as the CUDA stream, and every step of the
computation runs in the library's sm_100a kernels.  There is no CPU path: if
the library is missing or a call fails, an exception is raised.

Method: Flash Communication (sciencestack.ai/paper/2412.04964, TL;DR, Fig. 3-5)
-- per-block asymmetric INT8/INT4 quantization of tensor-parallel partial
sums, then a reduce-scatter (dequantize every rank's chunk, sum in fp32 in
rank order, requantize) and an all-gather (dequantize to fp16/bf16).  Here the
P ranks are P buffers on one GPU.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfc.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "fc.h")

FC_OK = 0
FC_ERR_INVALID_ARG = 1
FC_ERR_UNSUPPORTED = 2
FC_ERR_MISALIGNED = 3
FC_ERR_CUDA = 4
FC_ERR_TOO_LARGE = 5

# bytes of static device scratch behind fc_p2p_allreduce_emulated_noalloc
FC_NOALLOC_SCRATCH_BYTES = 16 << 20

FC_FP16 = 0
FC_BF16 = 1


class fc_qbuf(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("zps", ctypes.c_void_p)]


class FCError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        self.cuda_error = _lib().fc_last_cuda_error() if status == FC_ERR_CUDA else 0
        msg = f"{what}: {fc_status_string(status)}"
        if self.cuda_error:
            msg += f" (cudaError {self.cuda_error})"
        super().__init__(msg)


_LIB = None


def _lib():
    """Load libfc.so (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m bit_quantized_all_block_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        P, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        QP = ctypes.POINTER(fc_qbuf)
        L.fc_payload_sizes.argtypes = [S, I, I, ctypes.POINTER(S), ctypes.POINTER(S)]
        L.fc_quantize.argtypes = [P, I, S, I, I, QP, P]
        L.fc_rs_dequant_sum_requant.argtypes = [QP, I, S, I, I, QP, P]
        L.fc_ag_dequant.argtypes = [QP, S, I, I, I, P, P]
        L.fc_quantized_allreduce.argtypes = [ctypes.POINTER(P), I, I, S, I, I, P, QP, QP, P]
        L.fc_quantized_allreduce_ex.argtypes = [ctypes.POINTER(P), I, I, S, I, I, I, P, QP, QP, P]
        L.fc_gemm_quantize.argtypes = [P, P, I, I, I, I, I, I, QP, P, P, P]
        for f in ("fc_payload_sizes", "fc_quantize", "fc_rs_dequant_sum_requant", "fc_ag_dequant",
                  "fc_quantized_allreduce", "fc_quantized_allreduce_ex", "fc_gemm_quantize"):
            getattr(L, f).restype = I
        PP = ctypes.POINTER(P)
        L.fc_p2p_allreduce.argtypes = [I, I, I, S, I, I, P, P, QP, QP, PP, PP, ctypes.c_uint, P, I, P]
        L.fc_p2p_allreduce_emulated.argtypes = [I, I, S, I, I, PP, PP, QP, QP, PP, PP, ctypes.c_uint, P, I, P]
        L.fc_p2p_allreduce.restype = I
        L.fc_p2p_allreduce_emulated.restype = I
        L.fc_p2p_allreduce_emulated_noalloc.argtypes = [I, I, S, I, I, PP, PP, P, P]
        L.fc_p2p_allreduce_emulated_noalloc.restype = I
        L.fc_host_device_pointer.argtypes = [P, ctypes.POINTER(P)]
        L.fc_host_device_pointer.restype = I
        L.fc_ipc_export.argtypes = [P, ctypes.c_char_p, ctypes.POINTER(S)]
        L.fc_ipc_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(P)]
        L.fc_ipc_close.argtypes = [P]
        for f in ("fc_ipc_export", "fc_ipc_open", "fc_ipc_close"):
            getattr(L, f).restype = I
        L.fc_status_string.argtypes = [I]
        L.fc_status_string.restype = ctypes.c_char_p
        L.fc_last_cuda_error.argtypes = []
        L.fc_last_cuda_error.restype = I
        _LIB = L
    return _LIB


def library():
    """The loaded ctypes library (for callers that want the raw C ABI)."""
    return _lib()


def declared_symbols() -> list[str]:
    """Names of the functions include/fc.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:fc_status|const char\*|int)\s+(fc_\w+)\s*\(", text, re.M)))


def fc_status_string(status: int) -> str:
    return _lib().fc_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != FC_OK:
        raise FCError(status, what)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return FC_FP16
    if t.dtype == torch.bfloat16:
        return FC_BF16
    raise TypeError(f"expected float16 or bfloat16, got {t.dtype}")


def _torch_dtype(code: int):
    import torch
    return torch.float16 if code == FC_FP16 else torch.bfloat16


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev_ptr(t, name: str) -> int:
    """Device address of a contiguous CUDA tensor, or of a contiguous page-locked
    CPU tensor (the kernels then access host memory directly)."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.is_cuda:
        return t.data_ptr()
    if t.device.type == "cpu" and t.is_pinned():
        return fc_host_device_pointer(t.data_ptr())
    raise ValueError(f"{name} must be a CUDA tensor or a page-locked (pinned) CPU tensor")


def fc_host_device_pointer(host_ptr: int) -> int:
    """Device address of mapped page-locked host memory at ``host_ptr``."""
    d = ctypes.c_void_p()
    _check(_lib().fc_host_device_pointer(ctypes.c_void_p(host_ptr), ctypes.byref(d)), "fc_host_device_pointer")
    return d.value


def _new_like(t, n: int):
    """An output of n elements next to t: on its GPU, or page-locked if t is a pinned CPU tensor."""
    import torch
    if t.is_cuda:
        return torch.empty(n, dtype=t.dtype, device=t.device)
    return torch.empty(n, dtype=t.dtype).pin_memory()


def fc_payload_sizes(n: int, bits: int, block: int) -> tuple[int, int]:
    cb, nb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib().fc_payload_sizes(n, bits, block, ctypes.byref(cb), ctypes.byref(nb)), "fc_payload_sizes")
    return cb.value, nb.value


class QBuf:
    """A payload in device memory: packed codes (uint8), fp32 scales, uint8 zero-points."""

    def __init__(self, codes, scales, zps, n: int, bits: int, block: int):
        self.codes, self.scales, self.zps = codes, scales, zps
        self.n, self.bits, self.block = n, bits, block

    @classmethod
    def empty(cls, n: int, bits: int, block: int, device="cuda"):
        import torch
        cb, nb = fc_payload_sizes(n, bits, block)
        return cls(torch.empty(cb, dtype=torch.uint8, device=device),
                   torch.empty(nb, dtype=torch.float32, device=device),
                   torch.empty(nb, dtype=torch.uint8, device=device), n, bits, block)

    def struct(self) -> fc_qbuf:
        return fc_qbuf(_dev_ptr(self.codes, "codes"), _dev_ptr(self.scales, "scales"),
                       _dev_ptr(self.zps, "zps"))

    def bytes(self) -> int:
        return self.codes.numel() + 4 * self.scales.numel() + self.zps.numel()


class PeerQBuf(QBuf):
    """A payload held by another process's GPU, seen through fc_ipc_open
    mappings: raw device addresses instead of tensors."""

    def __init__(self, codes: int, scales: int, zps: int, n: int, bits: int, block: int):
        self.codes, self.scales, self.zps = codes, scales, zps
        self.n, self.bits, self.block = n, bits, block

    def struct(self):
        return fc_qbuf(self.codes, self.scales, self.zps)

    def bytes(self) -> int:
        cb, nb = fc_payload_sizes(self.n, self.bits, self.block)
        return cb + 5 * nb


FC_IPC_HANDLE_BYTES = 64


def fc_ipc_export(ptr: int) -> tuple[bytes, int]:
    """(IPC handle of the allocation holding device address ``ptr``, ptr's offset in it)."""
    h = ctypes.create_string_buffer(FC_IPC_HANDLE_BYTES)
    off = ctypes.c_size_t()
    _check(_lib().fc_ipc_export(ctypes.c_void_p(ptr), h, ctypes.byref(off)), "fc_ipc_export")
    return h.raw, off.value


def fc_ipc_open(handle: bytes) -> int:
    """Map another process's exported allocation; returns the base address."""
    if len(handle) != FC_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is 64 bytes")
    base = ctypes.c_void_p()
    _check(_lib().fc_ipc_open(handle, ctypes.byref(base)), "fc_ipc_open")
    return base.value


def fc_ipc_close(base: int) -> None:
    _check(_lib().fc_ipc_close(ctypes.c_void_p(base)), "fc_ipc_close")


def _addr(v) -> int:
    """Device address of a tensor or of a raw address."""
    return v if isinstance(v, int) else _dev_ptr(v, "pointer")


def _p2p_tables(P, s1, s2, ctr1, ctr2):
    if len(s1) != P * P or len(s2) != P or len(ctr1) != P or len(ctr2) != P:
        raise ValueError("s1 holds P*P payloads (s1[p*P + c]); s2, ctr1, ctr2 hold P entries")
    return ((fc_qbuf * (P * P))(*[q.struct() for q in s1]), (fc_qbuf * P)(*[q.struct() for q in s2]),
            (ctypes.c_void_p * P)(*[_addr(c) for c in ctr1]), (ctypes.c_void_p * P)(*[_addr(c) for c in ctr2]))


class P2PTables:
    """The payload and counter tables of fc_p2p_allreduce / fc_p2p_allreduce_emulated,
    marshalled once, for callers that call them many times on the same buffers (the
    arena of a collective object): building P*P payload descriptors costs tens to
    hundreds of microseconds of host time, more than a decode-sized call takes on
    the GPU."""

    def __init__(self, s1, s2, ctr1, ctr2):
        self.P = len(s2)
        self.args = _p2p_tables(self.P, s1, s2, ctr1, ctr2)
        # the tables hold raw addresses: keep the tensors behind them allocated
        self._keep = (list(s1), list(s2), list(ctr1), list(ctr2))


def fc_p2p_allreduce(rank: int, x, y, bits: int, block: int, s1, s2, ctr1, ctr2, epoch: int, status,
                     ctas_per_rank: int = 0, stream=None, tables: P2PTables | None = None):
    """One rank's one-kernel P-GPU all-reduce (see include/fc.h): s1 = P*P payloads (rank p's
    chunk c at p*P + c), s2 = P owners' payloads, ctr1/ctr2 = P counters (tensors or addresses);
    or `tables`, the same four marshalled once (s1, s2, ctr1, ctr2 are then not read).
    epoch: k for the k-th call on the counters, or 0 to let the kernel derive it (required for
    a call that a CUDA graph replays)."""
    if tables is None:
        tables = P2PTables(s1, s2, ctr1, ctr2)
    P = tables.P
    a1, a2, c1, c2 = tables.args
    _check(_lib().fc_p2p_allreduce(rank, P, _dtype_code(x), x.numel(), bits, block,
                                   ctypes.c_void_p(_dev_ptr(x, "x")), ctypes.c_void_p(_dev_ptr(y, "y")),
                                   a1, a2, c1, c2, epoch, ctypes.c_void_p(_addr(status)), ctas_per_rank,
                                   _stream(stream)), "fc_p2p_allreduce")
    return y


def fc_p2p_allreduce_emulated(xs, ys, bits: int, block: int, s1, s2, ctr1, ctr2, epoch: int, status,
                              ctas_per_rank: int = 0, stream=None, tables: P2PTables | None = None):
    """All P ranks of fc_p2p_allreduce in one cooperative launch on the current GPU."""
    P = len(xs)
    if tables is None:
        tables = P2PTables(s1, s2, ctr1, ctr2)
    if tables.P != P:
        raise ValueError("the tables are for another number of ranks")
    a1, a2, c1, c2 = tables.args
    xp = (ctypes.c_void_p * P)(*[_dev_ptr(x, "x") for x in xs])
    yp = (ctypes.c_void_p * P)(*[_dev_ptr(y, "y") for y in ys])
    _check(_lib().fc_p2p_allreduce_emulated(P, _dtype_code(xs[0]), xs[0].numel(), bits, block, xp, yp, a1, a2,
                                            c1, c2, epoch, ctypes.c_void_p(_addr(status)), ctas_per_rank,
                                            _stream(stream)), "fc_p2p_allreduce_emulated")
    return ys


def fc_p2p_allreduce_emulated_noalloc(xs, ys, bits: int, block: int, status=None, stream=None):
    """fc_p2p_allreduce_emulated with its payloads and counters in the library's static
    device scratch, for callers that must not allocate device memory (include/fc.h).
    ``ys`` are the P caller-owned outputs; ``status`` an optional device int (tensor or address)."""
    P = len(xs)
    if len(ys) != P:
        raise ValueError("xs and ys hold one tensor per rank")
    xp = (ctypes.c_void_p * P)(*[_dev_ptr(x, "x") for x in xs])
    yp = (ctypes.c_void_p * P)(*[_dev_ptr(y, "y") for y in ys])
    st = ctypes.c_void_p(_addr(status)) if status is not None else None
    _check(_lib().fc_p2p_allreduce_emulated_noalloc(P, _dtype_code(xs[0]), xs[0].numel(), bits, block, xp, yp, st,
                                                    _stream(stream)), "fc_p2p_allreduce_emulated_noalloc")
    return ys


def fc_quantize(x, bits: int, block: int, out: QBuf | None = None, stream=None) -> QBuf:
    """Step 1 on one rank: quantize the fp16/bf16 tensor x (flattened)."""
    n = x.numel()
    out = out or QBuf.empty(n, bits, block, x.device if x.is_cuda else "cuda")
    q = out.struct()
    _check(_lib().fc_quantize(ctypes.c_void_p(_dev_ptr(x, "x")), _dtype_code(x), n, bits, block,
                              ctypes.byref(q), _stream(stream)), "fc_quantize")
    return out


def fc_rs_dequant_sum_requant(ins, bits: int, block: int, out: QBuf | None = None, stream=None) -> QBuf:
    """Reduce-scatter step over the P step-1 payloads ``ins``; returns the step-2 payload."""
    P = len(ins)
    n = ins[0].n
    out = out or QBuf.empty(n, bits, block, ins[0].codes.device if hasattr(ins[0].codes, "device") else "cuda")
    arr = (fc_qbuf * P)(*[q.struct() for q in ins])
    q2 = out.struct()
    _check(_lib().fc_rs_dequant_sum_requant(arr, P, n, bits, block, ctypes.byref(q2), _stream(stream)),
           "fc_rs_dequant_sum_requant")
    return out


def fc_ag_dequant(q: QBuf, out_dtype, y=None, stream=None):
    """All-gather step: dequantize the step-2 payload to fp16/bf16 (``out_dtype`` a torch dtype)."""
    import torch
    code = FC_FP16 if out_dtype == torch.float16 else FC_BF16 if out_dtype == torch.bfloat16 else None
    if code is None:
        raise TypeError(f"out_dtype must be float16 or bfloat16, got {out_dtype}")
    if y is None:
        dev = q.codes.device if hasattr(q.codes, "device") else "cuda"
        y = torch.empty(q.n, dtype=out_dtype, device=dev)
    qs = q.struct()
    _check(_lib().fc_ag_dequant(ctypes.byref(qs), q.n, q.bits, q.block, code,
                                ctypes.c_void_p(_dev_ptr(y, "y")), _stream(stream)), "fc_ag_dequant")
    return y


def fc_quantized_allreduce(xs, bits: int, block: int, y=None, step1=None, step2: QBuf | None = None,
                           stream=None):
    """Fused two-step quantized all-reduce of the P partials ``xs`` (same shape and dtype).

    ``step1`` (a list of P QBufs) and ``step2`` optionally receive the wire payloads."""
    import torch
    P = len(xs)
    n = xs[0].numel()
    dt = _dtype_code(xs[0])
    for x in xs:
        if x.numel() != n or _dtype_code(x) != dt:
            raise ValueError("all partials must have the same size and dtype")
    y = _new_like(xs[0], n) if y is None else y
    xp = (ctypes.c_void_p * P)(*[_dev_ptr(x, "x") for x in xs])
    s1 = (fc_qbuf * P)(*[q.struct() for q in step1]) if step1 is not None else None
    s2 = step2.struct() if step2 is not None else None
    _check(_lib().fc_quantized_allreduce(xp, P, dt, n, bits, block, ctypes.c_void_p(_dev_ptr(y, "y")),
                                         s1, ctypes.byref(s2) if s2 is not None else None,
                                         _stream(stream)), "fc_quantized_allreduce")
    return y


def fc_quantized_allreduce_ex(xs, bits_rs: int, bits_ag: int, block: int, y=None, step1=None,
                              step2: QBuf | None = None, stream=None):
    """Fused all-reduce with a width per step (4, 8 or 16 = unquantized step)."""
    import torch
    P = len(xs)
    n = xs[0].numel()
    dt = _dtype_code(xs[0])
    for x in xs:
        if x.numel() != n or _dtype_code(x) != dt:
            raise ValueError("all partials must have the same size and dtype")
    y = _new_like(xs[0], n) if y is None else y
    xp = (ctypes.c_void_p * P)(*[_dev_ptr(x, "x") for x in xs])
    s1 = (fc_qbuf * P)(*[q.struct() for q in step1]) if step1 is not None else None
    s2 = step2.struct() if step2 is not None else None
    _check(_lib().fc_quantized_allreduce_ex(xp, P, dt, n, bits_rs, bits_ag, block,
                                            ctypes.c_void_p(_dev_ptr(y, "y")), s1,
                                            ctypes.byref(s2) if s2 is not None else None,
                                            _stream(stream)), "fc_quantized_allreduce_ex")
    return y


class PreparedAllReduce:
    """fc_quantized_allreduce_ex on fixed buffers, with its arguments marshalled once.

    For a caller that runs the same all-reduce on the same buffers many times
    outside a CUDA graph (a decode loop issuing one call per layer): building
    the ctypes arrays of device pointers costs more host time than a
    decode-sized kernel takes on the GPU (about 12-18 us against 2.5-3.4 us on
    B200), so they are built here once and each call only passes them to the C
    entry point: about 9 us a call, 5 of them in the entry point's own
    validation and launch.  The
    tensors' storage must stay where it is while the object is in use; their
    contents may change between calls.  ``stream``: a fixed stream for every
    call, or None for torch's current stream at each call."""

    def __init__(self, xs, bits_rs: int, bits_ag: int, block: int, y=None, step1=None,
                 step2: QBuf | None = None, stream=None):
        P = len(xs)
        n = xs[0].numel()
        dt = _dtype_code(xs[0])
        for x in xs:
            if x.numel() != n or _dtype_code(x) != dt:
                raise ValueError("all partials must have the same size and dtype")
        if step1 is not None and len(step1) != P:
            raise ValueError("step1 holds one payload per partial")
        self.y = _new_like(xs[0], n) if y is None else y
        self._keep = (list(xs), step1, step2)      # the buffers whose addresses are baked in
        xp = (ctypes.c_void_p * P)(*[_dev_ptr(x, "x") for x in xs])
        s1 = (fc_qbuf * P)(*[q.struct() for q in step1]) if step1 is not None else None
        self._s2 = step2.struct() if step2 is not None else None
        self._args = (xp, P, dt, n, bits_rs, bits_ag, block, ctypes.c_void_p(_dev_ptr(self.y, "y")), s1,
                      ctypes.byref(self._s2) if self._s2 is not None else None)
        self._stream = _stream(stream) if stream is not None else None
        self._fn = _lib().fc_quantized_allreduce_ex

    def __call__(self, stream=None):
        # (a fixed stream may be the legacy default stream, handle 0: test for None, not truth)
        if stream is not None:
            st = _stream(stream)
        elif self._stream is not None:
            st = self._stream
        else:
            st = _stream(None)
        status = self._fn(*self._args, st)
        if status != FC_OK:
            raise FCError(status, "fc_quantized_allreduce_ex")
        return self.y


def fc_gemm_quantize(a, w, bits: int, block: int, out: QBuf | None = None, partial=None, status=None,
                     quantize: bool = True, stream=None):
    """One rank's partial a @ w.T (tensor cores, fp32 accumulate, rounded to a.dtype) with the
    step-1 quantizer fused into the epilogue.

    Returns (payload or None, partial or None, status tensor).  ``quantize=False`` skips the
    payload (plain GEMM writing the partial); pass ``partial`` to also receive the partial."""
    import torch
    M, K = a.shape
    N, K2 = w.shape
    if K != K2 or a.dtype != w.dtype:
        raise ValueError("a is [M x K], w is [N x K], same dtype")
    dt = _dtype_code(a)
    if quantize and out is None:
        out = QBuf.empty(M * N, bits, block, a.device)
    if not quantize:
        out = None
        if partial is None:
            partial = torch.empty(M, N, dtype=a.dtype, device=a.device)
    status = torch.zeros(4, dtype=torch.int32, device=a.device) if status is None else status
    q = out.struct() if out is not None else None
    _check(_lib().fc_gemm_quantize(ctypes.c_void_p(_dev_ptr(a, "a")), ctypes.c_void_p(_dev_ptr(w, "w")), dt,
                                   M, N, K, bits, block, ctypes.byref(q) if q is not None else None,
                                   ctypes.c_void_p(_dev_ptr(partial, "partial")) if partial is not None else None,
                                   ctypes.c_void_p(_dev_ptr(status, "status")), _stream(stream)),
           "fc_gemm_quantize")
    return out, partial, status

