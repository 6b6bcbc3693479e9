"""The overlap check behind every entry point (a sort-and-sweep over the
call's ranges), fuzzed on the host: random layouts of the fused all-reduce's
and the one-kernel all-reduce's buffers in which exactly one written buffer
overlaps another buffer (output or input, any position, any order of
addresses) must be refused with FC_ERR_INVALID_ARG, and everything else about
the layout is valid (aligned, non-NULL), so the refusal can only come from the
overlap check.  Layouts without an overlap would pass validation and launch,
so none is ever passed; and the test does not run where a GPU is present,
where a missed overlap would launch a kernel on the fake addresses."""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="host-only: fake device addresses")

BASE = 0x100000000
GAP = 1 << 24


def _layout(rng, sizes):
    """Disjoint, 256-aligned ranges of the given sizes in random address order."""
    order = rng.permutation(len(sizes))
    addr = [0] * len(sizes)
    cur = BASE
    for i in order:
        addr[i] = cur
        cur += (sizes[i] + 255) // 256 * 256 + 256 * int(rng.integers(0, 64))
    return addr


def _overlap_one(rng, addr, sizes, writable):
    """Move one written range so that it overlaps another range (16-aligned start)."""
    i = int(rng.choice(writable))
    j = int(rng.choice([k for k in range(len(sizes)) if k != i]))
    # a 16-aligned start s with s < a_j + size_j and s + size_i > a_j; a_j itself
    # (256-aligned) always qualifies
    lo = -((-(addr[j] - sizes[i] + 1)) // 16)
    hi = (addr[j] + sizes[j] - 1) // 16
    addr[i] = 16 * int(rng.integers(lo, hi + 1))
    return i, j


def test_fused_allreduce_overlaps_are_refused():
    lib = fc.library()
    rng = np.random.default_rng(7)
    for trial in range(400):
        P = int(rng.integers(1, 9))
        block = int(rng.choice([32, 128, 1024]))
        n = P * block * int(rng.integers(1, 5))
        bits = int(rng.choice([4, 8]))
        nb, cb = n // block, n * bits // 8
        with_payloads = bool(rng.integers(0, 2))
        # ranges: P inputs, y, then (P step-1 + 1 step-2 payloads) x (codes, scales, zps)
        sizes = [2 * n] * P + [2 * n]
        if with_payloads:
            sizes += [cb, 4 * nb, nb] * (P + 1)
        writable = list(range(P, len(sizes)))
        addr = _layout(rng, sizes)
        _overlap_one(rng, addr, sizes, writable)
        xp = (ctypes.c_void_p * P)(*addr[:P])
        y = ctypes.c_void_p(addr[P])
        s1 = s2 = None
        if with_payloads:
            q = [fc.fc_qbuf(*addr[P + 1 + 3 * i: P + 4 + 3 * i]) for i in range(P + 1)]
            s1 = (fc.fc_qbuf * P)(*q[:P])
            s2 = ctypes.byref(q[P])
        st = lib.fc_quantized_allreduce_ex(xp, P, 0, n, bits, bits, block, y, s1, s2, None)
        assert st == fc.FC_ERR_INVALID_ARG, (trial, P, block, n, with_payloads, st)


def test_one_kernel_allreduce_overlaps_are_refused():
    lib = fc.library()
    rng = np.random.default_rng(8)
    for trial in range(200):
        P = int(rng.choice([2, 4, 8]))
        block = int(rng.choice([32, 128]))
        n = P * block * int(rng.integers(1, 4))
        m = n // P
        nb, cb = m // block, m * 8 // 8
        # ranges: P inputs, P outputs, P*P + P payloads (3 each), 2P counters, status
        sizes = [2 * n] * P + [2 * n] * P + [cb, 4 * nb, nb] * (P * P + P) + [4] * (2 * P) + [4]
        writable = list(range(P, len(sizes)))
        first_counter = 2 * P + 3 * (P * P + P)
        addr = _layout(rng, sizes)
        i, j = _overlap_one(rng, addr, sizes, writable)
        if i >= first_counter and rng.integers(0, 2):   # counters and status need only 4-byte alignment
            addr[i] = addr[j] + 4 * int(rng.integers(0, max(1, sizes[j] // 4)))
        xp = (ctypes.c_void_p * P)(*addr[:P])
        yp = (ctypes.c_void_p * P)(*addr[P:2 * P])
        k = 2 * P
        q = [fc.fc_qbuf(*addr[k + 3 * t: k + 3 * t + 3]) for t in range(P * P + P)]
        k += 3 * (P * P + P)
        s1 = (fc.fc_qbuf * (P * P))(*q[:P * P])
        s2 = (fc.fc_qbuf * P)(*q[P * P:])
        c1 = (ctypes.c_void_p * P)(*addr[k:k + P])
        c2 = (ctypes.c_void_p * P)(*addr[k + P:k + 2 * P])
        status = ctypes.c_void_p(addr[k + 2 * P])
        st = lib.fc_p2p_allreduce_emulated(P, 0, n, 8, block, xp, yp, s1, s2, c1, c2, 1, status, 0, None)
        assert st == fc.FC_ERR_INVALID_ARG, (trial, P, block, n, i, j, st)
