"""The C-ABI library loads on the host and exports everything include/fc.h
declares; host-only entry points and host-side validation behave as
documented.  No call here reaches a CUDA API: every validation case fails
before launch (fake, never-dereferenced pointer values are used)."""
import ctypes

import pytest

import bit_quantized_all_block_b200 as fc


def test_library_exports_every_declared_symbol():
    names = fc.declared_symbols()
    assert set(names) >= {"fc_payload_sizes", "fc_quantize", "fc_rs_dequant_sum_requant",
                          "fc_ag_dequant", "fc_quantized_allreduce", "fc_status_string",
                          "fc_last_cuda_error"}
    lib = fc.library()
    for n in names:
        assert hasattr(lib, n), n


def test_payload_sizes():
    assert fc.fc_payload_sizes(8192 * 8192, 8, 128) == (8192 * 8192, 8192 * 64)
    assert fc.fc_payload_sizes(4096, 4, 4096) == (2048, 1)
    assert fc.fc_payload_sizes(0, 4, 32) == (0, 0)
    for n, bits, block in [(100, 8, 128), (256, 3, 128), (256, 8, 48), (256, 8, 16), (8192, 8, 8192)]:
        with pytest.raises(fc.FCError) as e:
            fc.fc_payload_sizes(n, bits, block)
        assert e.value.status == fc.FC_ERR_INVALID_ARG


def test_status_strings():
    for st in range(6):
        assert fc.fc_status_string(st)
    assert fc.library().fc_last_cuda_error() == 0


A = 0x10000000   # fake, 16-byte aligned device addresses (never dereferenced)


def qb(base):
    return fc.fc_qbuf(base, base + 0x1000000, base + 0x2000000)


def fused(x, P, n, bits=8, block=128, y=A + 0x40000000, step1=None, step2=None, dtype=0):
    lib = fc.library()
    xp = (ctypes.c_void_p * len(x))(*x)
    s1 = (fc.fc_qbuf * P)(*step1) if step1 is not None else None
    s2 = ctypes.byref(step2) if step2 is not None else None
    return lib.fc_quantized_allreduce(xp, P, dtype, n, bits, block, ctypes.c_void_p(y), s1, s2, None)


XS = [A + r * 0x1000000 for r in range(8)]


@pytest.mark.parametrize("kw,expect", [
    (dict(P=4, n=4096, bits=3), fc.FC_ERR_INVALID_ARG),
    (dict(P=4, n=4096, block=48), fc.FC_ERR_INVALID_ARG),
    (dict(P=4, n=4096, block=16), fc.FC_ERR_INVALID_ARG),
    (dict(P=4, n=4096 * 4, block=8192), fc.FC_ERR_INVALID_ARG),
    (dict(P=0, n=4096), fc.FC_ERR_INVALID_ARG),
    (dict(P=9, n=4096 * 9), fc.FC_ERR_INVALID_ARG),
    (dict(P=3, n=1024), fc.FC_ERR_INVALID_ARG),           # n % (P*block) != 0
    (dict(P=4, n=4096, dtype=2), fc.FC_ERR_INVALID_ARG),
    (dict(P=4, n=4096, y=A + 0x40000008), fc.FC_ERR_MISALIGNED),
    (dict(P=4, n=4096, y=0), fc.FC_ERR_INVALID_ARG),
    (dict(P=4, n=4096, y=XS[2] + 512), fc.FC_ERR_INVALID_ARG),   # y overlaps x[2]
    (dict(P=4, n=0, y=0), fc.FC_OK),                              # empty: no-op
])
def test_fused_validation(kw, expect):
    P = kw.pop("P")
    assert fused(XS[:max(P, 1)] if P <= 8 else XS + XS[:1], P, **kw) == expect


def test_fused_validation_pointers():
    x = list(XS[:4])
    x[1] = XS[1] + 4
    assert fused(x, 4, 4096) == fc.FC_ERR_MISALIGNED
    x[1] = 0
    assert fused(x, 4, 4096) == fc.FC_ERR_INVALID_ARG
    # payload outputs: overlapping each other, or misaligned
    s1 = [qb(A + 0x50000000 + r * 0x4000000) for r in range(4)]
    s1[3] = qb(A + 0x50000000)
    assert fused(XS[:4], 4, 4096, step1=s1) == fc.FC_ERR_INVALID_ARG
    s2 = fc.fc_qbuf(A + 0x70000000, A + 0x70000004, A + 0x71000000)
    assert fused(XS[:4], 4, 4096, step2=s2) == fc.FC_ERR_MISALIGNED
    s2 = fc.fc_qbuf(A + 0x70000000, 0, A + 0x71000000)
    assert fused(XS[:4], 4, 4096, step2=s2) == fc.FC_ERR_INVALID_ARG


def test_staged_validation():
    lib = fc.library()
    q = qb(A + 0x50000000)
    assert lib.fc_quantize(ctypes.c_void_p(A), 0, 4096, 5, 128, ctypes.byref(q), None) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_quantize(ctypes.c_void_p(A + 2), 0, 4096, 8, 128, ctypes.byref(q), None) == fc.FC_ERR_MISALIGNED
    assert lib.fc_quantize(ctypes.c_void_p(A), 0, 4000, 8, 128, ctypes.byref(q), None) == fc.FC_ERR_INVALID_ARG
    qo = qb(A)      # codes overlap x
    assert lib.fc_quantize(ctypes.c_void_p(A), 0, 4096, 8, 128, ctypes.byref(qo), None) == fc.FC_ERR_INVALID_ARG
    ins = (fc.fc_qbuf * 2)(qb(A), qb(A + 0x4000000))
    assert lib.fc_rs_dequant_sum_requant(ins, 2, 4096, 8, 128, ctypes.byref(ins[0]), None) == fc.FC_ERR_INVALID_ARG
    # any whole number of blocks is a valid range; a partial block is not
    assert lib.fc_rs_dequant_sum_requant(ins, 2, 4096 + 64, 8, 128, ctypes.byref(q), None) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_rs_dequant_sum_requant(ins, 2, 0, 8, 128, None, None) == fc.FC_OK
    assert lib.fc_ag_dequant(ctypes.byref(q), 4096, 8, 128, 0, ctypes.c_void_p(A + 0x50000000), None) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_ag_dequant(ctypes.byref(q), 4096, 8, 128, 0, ctypes.c_void_p(A + 0x7000000a), None) == fc.FC_ERR_MISALIGNED
    assert lib.fc_ag_dequant(ctypes.byref(q), 4096, 8, 128, 3, ctypes.c_void_p(A), None) == fc.FC_ERR_INVALID_ARG


def test_ipc_validation():
    lib = fc.library()
    h = ctypes.create_string_buffer(fc.FC_IPC_HANDLE_BYTES)
    off = ctypes.c_size_t()
    base = ctypes.c_void_p()
    assert lib.fc_ipc_export(None, h, ctypes.byref(off)) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_ipc_export(ctypes.c_void_p(A), None, ctypes.byref(off)) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_ipc_export(ctypes.c_void_p(A), h, None) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_ipc_open(None, ctypes.byref(base)) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_ipc_open(h, None) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_ipc_close(None) == fc.FC_ERR_INVALID_ARG
    dev = ctypes.c_void_p()
    assert lib.fc_host_device_pointer(None, ctypes.byref(dev)) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_host_device_pointer(ctypes.c_void_p(A), None) == fc.FC_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        fc.fc_ipc_open(b"short")


def test_p2p_validation():
    lib = fc.library()
    P = 2
    s1 = (fc.fc_qbuf * 4)(*[qb(A + i * 0x1000000) for i in range(4)])
    s2 = (fc.fc_qbuf * 2)(*[qb(A + (4 + i) * 0x1000000) for i in range(2)])
    ctr = (ctypes.c_void_p * 2)(A + 0x70000000, A + 0x70000010)
    st = ctypes.c_void_p(A + 0x70000100)
    x, y = ctypes.c_void_p(A + 0x60000000), ctypes.c_void_p(A + 0x68000000)
    call = lambda **kw: lib.fc_p2p_allreduce(kw.get("rank", 0), kw.get("P", P), 0, kw.get("n", 4096), kw.get("bits", 8),
                                             128, x, y, s1, s2, ctr, ctr, kw.get("epoch", 1), st, 0, None)
    assert call(P=3) == fc.FC_ERR_INVALID_ARG          # P in {2, 4, 8}
    assert call(rank=2) == fc.FC_ERR_INVALID_ARG
    assert call(bits=5) == fc.FC_ERR_INVALID_ARG
    assert call(n=4096 + 128) == fc.FC_ERR_INVALID_ARG  # n % (P*block)
    # (epoch 0 is valid: the kernel derives the epoch from the counters.  Every call
    # here must fail validation, since a call that passed it would launch on these
    # made-up addresses; epoch 0 is exercised on real buffers in test_gpu_p2p.py)
    assert call(n=0) == fc.FC_OK
    assert lib.fc_p2p_allreduce(0, 2, 0, 4096, 8, 128, x, y, None, s2, ctr, ctr, 1, st, 0, None) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_p2p_allreduce(0, 2, 0, 4096, 8, 128, x, y, s1, s2, ctr, ctr, 1, None, 0, None) == fc.FC_ERR_INVALID_ARG


def test_p2p_overlap_validation():
    """Buffers the one-kernel all-reduce writes may not overlap each other or its input."""
    lib = fc.library()
    P = 2
    ctr1 = (ctypes.c_void_p * 2)(A + 0x70000000, A + 0x70000010)
    ctr2 = (ctypes.c_void_p * 2)(A + 0x70000020, A + 0x70000030)
    x, y = A + 0x60000000, A + 0x68000000

    def call(s1_bases=None, s2_bases=None, st=A + 0x70000100, yy=y, c2=ctr2, emu=False):
        s1 = (fc.fc_qbuf * 4)(*[qb(b) for b in (s1_bases or [A + i * 0x100000 for i in range(4)])])
        s2 = (fc.fc_qbuf * 2)(*[qb(b) for b in (s2_bases or [A + 0x400000 + i * 0x100000 for i in range(2)])])
        if emu:
            xp = (ctypes.c_void_p * 2)(x, x + 0x10000)
            yp = (ctypes.c_void_p * 2)(yy, yy + 0x10000)
            return lib.fc_p2p_allreduce_emulated(P, 0, 4096, 8, 128, xp, yp, s1, s2, ctr1, c2, 1,
                                                 ctypes.c_void_p(st), 0, None)
        return lib.fc_p2p_allreduce(0, P, 0, 4096, 8, 128, ctypes.c_void_p(x), ctypes.c_void_p(yy), s1, s2,
                                    ctr1, c2, 1, ctypes.c_void_p(st), 0, None)

    for emu in (False, True):
        # two step-1 payloads share their codes
        assert call(s1_bases=[A, A, A + 0x200000, A + 0x300000], emu=emu) == fc.FC_ERR_INVALID_ARG
        # a step-2 payload's codes inside a step-1 payload's codes
        assert call(s2_bases=[A + 0x100, A + 0x500000], emu=emu) == fc.FC_ERR_INVALID_ARG
        # the output over the input, the status word on a counter, a counter on a counter
        assert call(yy=x + 0x100, emu=emu) == fc.FC_ERR_INVALID_ARG
        assert call(st=A + 0x70000010, emu=emu) == fc.FC_ERR_INVALID_ARG
        assert call(c2=(ctypes.c_void_p * 2)(A + 0x70000000, A + 0x70000030), emu=emu) == fc.FC_ERR_INVALID_ARG
    # emulated: one rank's output over another rank's output
    xp = (ctypes.c_void_p * 2)(x, x + 0x10000)
    yp = (ctypes.c_void_p * 2)(y, y + 0x100)
    s1 = (fc.fc_qbuf * 4)(*[qb(A + i * 0x100000) for i in range(4)])
    s2 = (fc.fc_qbuf * 2)(*[qb(A + 0x400000 + i * 0x100000) for i in range(2)])
    assert lib.fc_p2p_allreduce_emulated(P, 0, 4096, 8, 128, xp, yp, s1, s2, ctr1, ctr2, 1,
                                         ctypes.c_void_p(A + 0x70000100), 0, None) == fc.FC_ERR_INVALID_ARG


def test_noalloc_validation_before_any_cuda_call():
    """The entry point without allocation refuses bad arguments and problems larger than its
    static scratch on the host, before it looks up the scratch or launches anything."""
    lib = fc.library()

    def call(P, n, bits=8, block=128, dtype=0, x=XS, y=XS):
        xp = (ctypes.c_void_p * 8)(*x[:8])
        yp = (ctypes.c_void_p * 8)(*[a + 0x80000000 for a in y[:8]])
        return lib.fc_p2p_allreduce_emulated_noalloc(P, dtype, n, bits, block, xp, yp, None, None)

    assert call(4, 0) == fc.FC_OK
    assert call(3, 3 * 128) == fc.FC_ERR_INVALID_ARG
    assert call(4, 4 * 128 + 128) == fc.FC_ERR_INVALID_ARG
    assert call(4, 4 * 128, bits=6) == fc.FC_ERR_INVALID_ARG
    assert call(4, 4 * 128, dtype=2) == fc.FC_ERR_INVALID_ARG
    assert lib.fc_p2p_allreduce_emulated_noalloc(4, 0, 512, 8, 128, None, None, None, None) == fc.FC_ERR_INVALID_ARG
    assert call(4, 4 * 128 * 8192) == fc.FC_ERR_TOO_LARGE            # 4 Mi elements per rank at INT8
    assert call(8, 1 << 40) == fc.FC_ERR_TOO_LARGE


def _prototypes():
    """{name: [parameter declarations]} for every function include/fc.h declares."""
    import re
    text = open(fc.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"(?:fc_status|const char\*|int)\s+(fc_\w+)\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        protos[m.group(1)] = params
    return protos


def test_binding_signatures_match_the_header():
    """Every ctypes signature the binding sets has the header's arity, and each
    argument is a pointer exactly where the header declares one."""
    protos = _prototypes()
    assert set(protos) == set(fc.declared_symbols())
    lib = fc.library()
    pointer_types = (ctypes.c_void_p, ctypes.c_char_p)
    for name, params in protos.items():
        argtypes = getattr(lib, name).argtypes
        if argtypes is None:
            continue
        assert len(argtypes) == len(params), f"{name}: {len(argtypes)} ctypes arguments, header has {len(params)}"
        for decl, t in zip(params, argtypes):
            is_ptr = "*" in decl
            t_ptr = t in pointer_types or hasattr(t, "_type_") and issubclass(t, ctypes._Pointer)
            assert is_ptr == bool(t_ptr), f"{name}: '{decl}' bound as {t}"


def test_gemm_validation():
    """fc_gemm_quantize refuses bad shapes, block sizes, missing or misaligned buffers and
    outputs that overlap the operands -- all before any CUDA call."""
    lib = fc.library()
    a, w, part, st = A, A + 0x8000000, A + 0x10000000, A + 0x18000000
    out = qb(A + 0x20000000)

    def call(M=256, N=512, K=128, bits=8, block=128, a=a, w=w, out=out, part=part, st=st, dtype=0):
        return lib.fc_gemm_quantize(ctypes.c_void_p(a), ctypes.c_void_p(w), dtype, M, N, K, bits, block,
                                    ctypes.byref(out) if out is not None else None, ctypes.c_void_p(part)
                                    if part is not None else None, ctypes.c_void_p(st) if st is not None else None,
                                    None)

    for kw in (dict(M=100), dict(N=100), dict(K=100), dict(M=0), dict(block=512), dict(block=16),
               dict(bits=5), dict(dtype=2), dict(out=None, part=None), dict(st=None), dict(a=0)):
        assert call(**kw) == fc.FC_ERR_INVALID_ARG, kw
    assert call(a=a + 8) == fc.FC_ERR_MISALIGNED
    assert call(part=part + 4) == fc.FC_ERR_MISALIGNED
    assert call(st=st + 2) == fc.FC_ERR_MISALIGNED
    assert call(part=a + 0x1000) == fc.FC_ERR_INVALID_ARG          # partial overlaps a
    assert call(st=w) == fc.FC_ERR_INVALID_ARG                     # status overlaps w


def test_per_step_width_validation():
    """fc_quantized_allreduce_ex: widths outside {4, 8, 16}, a payload for an unquantized step,
    sizes that are not whole chunks, and the width combinations the library does not provide."""
    lib = fc.library()

    def call(P=4, n=4096, b1=8, b2=4, block=128, step1=None, step2=None):
        xp = (ctypes.c_void_p * P)(*XS[:P])
        s1 = (fc.fc_qbuf * P)(*step1) if step1 is not None else None
        return lib.fc_quantized_allreduce_ex(xp, P, 0, n, b1, b2, block, ctypes.c_void_p(A + 0x40000000), s1,
                                             ctypes.byref(step2) if step2 is not None else None, None)

    assert call(b1=5) == fc.FC_ERR_INVALID_ARG
    assert call(b2=12) == fc.FC_ERR_INVALID_ARG
    assert call(b1=16, step1=[qb(A + 0x50000000 + i * 0x4000000) for i in range(4)]) == fc.FC_ERR_INVALID_ARG
    assert call(b2=16, step2=qb(A + 0x60000000)) == fc.FC_ERR_INVALID_ARG
    assert call(n=4096 + 128) == fc.FC_ERR_INVALID_ARG
    assert call(P=3, n=3 * 128 * 4, b1=8, b2=4) == fc.FC_ERR_UNSUPPORTED
    assert call(P=3, n=3 * 128 * 4, b1=16, b2=16) == fc.FC_ERR_UNSUPPORTED
    assert call(n=0) == fc.FC_OK
