"""A second, vectorised numpy-float32 statement of the oracle's definition.

Cross-check only (test infrastructure): it restates the same readings, so it
catches slips in the C code (indexing, packing, loop bounds) but is not one of
the oracle's pins.  numpy float32 arithmetic rounds each operation to nearest
even; np.rint rounds half to even."""
import numpy as np

F32 = np.float32


def quantize(v32, bits, B):
    qmax = (1 << bits) - 1
    v = np.asarray(v32, F32).reshape(-1, B)
    mn = np.minimum(v.min(1), F32(0))
    mx = np.maximum(v.max(1), F32(0))
    d = (mx - mn).astype(F32)
    with np.errstate(divide="ignore"):
        s = np.where(d == 0, F32(1), d / F32(qmax)).astype(F32)
        inv = (F32(1) / s).astype(F32)
    # integer rounding of the exact product (exact in float64: 24 x 24 bits)
    f64 = np.float64
    z = np.clip(np.rint((-mn).astype(f64) * inv.astype(f64)), 0, qmax).astype(np.int64)
    q = np.clip(np.rint(v.astype(f64) * inv.astype(f64)[:, None]).astype(np.int64) + z[:, None], 0, qmax)
    return q.ravel(), s, z


def dequantize(q, s, z, B):
    qz = (q.reshape(-1, B) - z[:, None]).astype(F32)
    return (qz * s[:, None]).astype(F32).ravel()


def pack(q, bits):
    q = q.astype(np.uint8)
    if bits == 8:
        return q
    return (q[0::2] | (q[1::2] << 4)).astype(np.uint8)


def allreduce(v32s, bits, B):
    """v32s: P x n fp32 inputs (already widened).  Returns (q1s, s1s, z1s, q2, s2, z2, xhat2)."""
    q1s, s1s, z1s, xh = [], [], [], []
    for v in v32s:
        q, s, z = quantize(v, bits, B)
        q1s.append(q); s1s.append(s); z1s.append(z)
        xh.append(dequantize(q, s, z, B))
    acc = xh[0].copy()
    for r in range(1, len(xh)):
        acc = (acc + xh[r]).astype(F32)
    q2, s2, z2 = quantize(acc, bits, B)
    return q1s, s1s, z1s, q2, s2, z2, dequantize(q2, s2, z2, B)
