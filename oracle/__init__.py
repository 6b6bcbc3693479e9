"""CPU oracle for the low-bit two-step quantized all-reduce (Flash Communication).

TEST INFRASTRUCTURE ONLY.  This package wraps ``fco.c``, the plain scalar
definition the CUDA library is checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the library under ``bit_quantized_all_block_b200`` never does, and the two
share no code.

The method (Flash Communication, sciencestack.ai/paper/2412.04964, TL;DR and
Fig. 4-5): per-block asymmetric low-bit quantization of each rank's partial,
then a two-step all-reduce -- reduce-scatter (dequantize a chunk from every
rank, sum in fp32, requantize) and all-gather (dequantize to fp16/bf16).  The
exact arithmetic (a reading of the page, which gives no formulas) is written
out in the header comment of ``fco.c``.

Parity pins for every function here live in ``tests/test_oracle_*.py``:
hand-derived fixtures in ``tests/golden/``, brute force over tiny blocks,
the per-element error bound |x - xhat| <= s/2, exact round trips of
representable grids, invariants (P=1, power-of-two scaling, permutations,
zeros) and library references for the fp16/bf16 conversions.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fco.c")
_LIB = os.path.join(_HERE, "libfco.so")

FP16 = 0
BF16 = 1

OK = 0
ERR_ARG = 1
ERR_RANGE = 2

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile fco.c into libfco.so next to it (gcc, strict IEEE flags)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Temporarily route every wrapper through another build of fco.c (the
    mutation tests use this to show that the pins reject planted mistakes)."""
    global _lib
    saved = _lib
    _lib = _bind(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _bind(L):
    P = ctypes.c_void_p
    S = ctypes.c_size_t
    I = ctypes.c_int
    F = ctypes.c_float
    L.fco_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.fco_f16_to_f32.restype = F
    L.fco_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.fco_bf16_to_f32.restype = F
    L.fco_f32_to_f16.argtypes = [F]
    L.fco_f32_to_f16.restype = ctypes.c_uint16
    L.fco_f32_to_bf16.argtypes = [F]
    L.fco_f32_to_bf16.restype = ctypes.c_uint16
    L.fco_widen.argtypes = [P, I, S, P]
    L.fco_widen.restype = None
    L.fco_narrow.argtypes = [P, I, S, P]
    L.fco_narrow.restype = None
    L.fco_quantize_f32.argtypes = [P, S, I, I, P, P, P]
    L.fco_block_stats.argtypes = [P, I, I, P, P, P]
    L.fco_quantize_value.argtypes = [F, F, I, I]
    L.fco_dequantize_value.argtypes = [I, F, I]
    L.fco_dequantize_value.restype = F
    L.fco_quantize.argtypes = [P, I, S, I, I, P, P, P]
    L.fco_dequantize.argtypes = [P, P, P, S, I, I, P]
    L.fco_rs_dequant_sum_requant.argtypes = [P, P, P, I, S, I, I, P, P, P]
    L.fco_ag_dequant.argtypes = [P, P, P, S, I, I, I, P]
    L.fco_allreduce.argtypes = [P, I, I, S, I, I, P, P, P, P, P, P, P]
    L.fco_allreduce_ex.argtypes = [P, I, I, S, I, I, I, P, P, P, P, P, P, P]
    for name in ("fco_block_stats", "fco_quantize_value", "fco_quantize", "fco_quantize_f32",
                 "fco_dequantize",
                 "fco_rs_dequant_sum_requant", "fco_ag_dequant", "fco_allreduce", "fco_allreduce_ex"):
        getattr(L, name).restype = I
    return L


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _ptr_array(arrs):
    return (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])


def _check(st: int, what: str):
    if st != OK:
        raise OracleError(f"{what}: oracle status {st}")


def code_bytes(n: int, bits: int) -> int:
    return n * bits // 8


class Payload:
    """Host payload of one quantization: packed codes, fp32 scales, uint8 zero-points."""

    def __init__(self, n: int, bits: int, block: int):
        self.n, self.bits, self.block = n, bits, block
        self.codes = np.zeros(code_bytes(n, bits), dtype=np.uint8)
        nb = n // block if block > 0 else 0
        self.scales = np.zeros(nb, dtype=np.float32)
        self.zps = np.zeros(nb, dtype=np.uint8)


# -- scalar helpers -------------------------------------------------------------

def f16_to_f32(h: int) -> float:
    return lib().fco_f16_to_f32(int(h))


def bf16_to_f32(b: int) -> float:
    return lib().fco_bf16_to_f32(int(b))


def f32_to_f16(x: float) -> int:
    return lib().fco_f32_to_f16(float(x))


def f32_to_bf16(x: float) -> int:
    return lib().fco_f32_to_bf16(float(x))


def block_stats(v: np.ndarray, bits: int):
    """(s, inv, z) of one block of fp32 values."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    s = np.zeros(1, np.float32)
    inv = np.zeros(1, np.float32)
    z = np.zeros(1, np.int32)
    _check(lib().fco_block_stats(_ptr(v), len(v), bits, _ptr(s), _ptr(inv), _ptr(z)), "block_stats")
    return np.float32(s[0]), np.float32(inv[0]), int(z[0])


def quantize_value(v: float, inv: float, z: int, bits: int) -> int:
    return lib().fco_quantize_value(float(v), float(inv), int(z), bits)


def dequantize_value(q: int, s: float, z: int) -> np.float32:
    return np.float32(lib().fco_dequantize_value(int(q), float(s), int(z)))


# -- array entry points --------------------------------------------------------

def widen(x_u16: np.ndarray, dtype: int) -> np.ndarray:
    """Exact widening of fp16/bf16 bit patterns to fp32."""
    x = np.ascontiguousarray(x_u16, dtype=np.uint16).ravel()
    out = np.zeros(x.size, dtype=np.float32)
    lib().fco_widen(_ptr(x), dtype, x.size, _ptr(out))
    return out


def narrow(v: np.ndarray, dtype: int) -> np.ndarray:
    """fp32 -> fp16/bf16 bit patterns, round to nearest, ties to even."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.zeros(v.size, dtype=np.uint16)
    lib().fco_narrow(_ptr(v), dtype, v.size, _ptr(out))
    return out


def quantize_f32(v: np.ndarray, bits: int, block: int) -> Payload:
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    p = Payload(v.size, bits, block)
    _check(lib().fco_quantize_f32(_ptr(v), v.size, bits, block,
                                  _ptr(p.codes), _ptr(p.scales), _ptr(p.zps)), "quantize_f32")
    return p


def quantize(x_u16: np.ndarray, dtype: int, bits: int, block: int) -> Payload:
    x = np.ascontiguousarray(x_u16, dtype=np.uint16).ravel()
    p = Payload(x.size, bits, block)
    _check(lib().fco_quantize(_ptr(x), dtype, x.size, bits, block,
                              _ptr(p.codes), _ptr(p.scales), _ptr(p.zps)), "quantize")
    return p


def dequantize(p: Payload) -> np.ndarray:
    out = np.zeros(p.n, dtype=np.float32)
    _check(lib().fco_dequantize(_ptr(p.codes), _ptr(p.scales), _ptr(p.zps), p.n, p.bits,
                                p.block, _ptr(out)), "dequantize")
    return out


def rs_dequant_sum_requant(payloads) -> Payload:
    P = len(payloads)
    p0 = payloads[0]
    out = Payload(p0.n, p0.bits, p0.block)
    _check(lib().fco_rs_dequant_sum_requant(
        _ptr_array([p.codes for p in payloads]), _ptr_array([p.scales for p in payloads]),
        _ptr_array([p.zps for p in payloads]), P, p0.n, p0.bits, p0.block,
        _ptr(out.codes), _ptr(out.scales), _ptr(out.zps)), "rs_dequant_sum_requant")
    return out


def ag_dequant(p: Payload, out_dtype: int) -> np.ndarray:
    y = np.zeros(p.n, dtype=np.uint16)
    _check(lib().fco_ag_dequant(_ptr(p.codes), _ptr(p.scales), _ptr(p.zps), p.n, p.bits,
                                p.block, out_dtype, _ptr(y)), "ag_dequant")
    return y


def allreduce(xs, dtype: int, bits: int, block: int):
    """Whole two-step all-reduce.  xs: list of P uint16 arrays (fp16/bf16 bits).

    Returns (y, step1 payloads, step2 payload)."""
    xs = [np.ascontiguousarray(x, dtype=np.uint16).ravel() for x in xs]
    P, n = len(xs), xs[0].size
    p1 = [Payload(n, bits, block) for _ in range(P)]
    p2 = Payload(n, bits, block)
    y = np.zeros(n, dtype=np.uint16)
    _check(lib().fco_allreduce(_ptr_array(xs), P, dtype, n, bits, block,
                               _ptr_array([p.codes for p in p1]), _ptr_array([p.scales for p in p1]),
                               _ptr_array([p.zps for p in p1]),
                               _ptr(p2.codes), _ptr(p2.scales), _ptr(p2.zps), _ptr(y)), "allreduce")
    return y, p1, p2


def allreduce_ex(xs, dtype: int, bits_rs: int, bits_ag: int, block: int):
    """Two-step all-reduce with per-step precision (4, 8 or 16 = unquantized).

    Returns (y, step1 payloads or None, step2 payload or None)."""
    xs = [np.ascontiguousarray(x, dtype=np.uint16).ravel() for x in xs]
    P, n = len(xs), xs[0].size
    b1 = bits_rs if bits_rs != 16 else 8
    b2 = bits_ag if bits_ag != 16 else 8
    p1 = [Payload(n, b1, block) for _ in range(P)]
    p2 = Payload(n, b2, block)
    y = np.zeros(n, dtype=np.uint16)
    _check(lib().fco_allreduce_ex(_ptr_array(xs), P, dtype, n, bits_rs, bits_ag, block,
                                  _ptr_array([p.codes for p in p1]), _ptr_array([p.scales for p in p1]),
                                  _ptr_array([p.zps for p in p1]),
                                  _ptr(p2.codes), _ptr(p2.scales), _ptr(p2.zps), _ptr(y)), "allreduce_ex")
    return y, (p1 if bits_rs != 16 else None), (p2 if bits_ag != 16 else None)

