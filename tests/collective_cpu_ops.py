"""Host stand-in for the device side of `collective.QuantizedAllReduce`, for
the multi-process CPU tests (test infrastructure): arenas are POSIX shared
memory, shared between the rank processes the way peer mappings share GPU
memory, and each step is the CPU oracle's step on views into the arenas."""
from multiprocessing import shared_memory

import numpy as np

import oracle


class OracleOps:
    def __init__(self, dtype: int):
        self.dtype = dtype
        self.shm = None
        self.peers = {}

    def alloc(self, nbytes: int):
        self.shm = shared_memory.SharedMemory(create=True, size=max(nbytes, 256))

    def export(self):
        return self.shm.name

    def device_id(self) -> str:
        return "cpu"

    def attach(self, rank: int, exported: list):
        for r, name in enumerate(exported):
            self.peers[r] = self.shm if r == rank else shared_memory.SharedMemory(name=name)

    def payload(self, ref, bits: int, block: int) -> oracle.Payload:
        buf = self.peers[ref.holder].buf
        p = oracle.Payload(0, bits, block)
        p.n = ref.n
        cb, nb = oracle.code_bytes(ref.n, bits), ref.n // block
        p.codes = np.ndarray((cb,), np.uint8, buf, ref.codes)
        p.scales = np.ndarray((nb,), np.float32, buf, ref.scales)
        p.zps = np.ndarray((nb,), np.uint8, buf, ref.zps)
        return p

    @staticmethod
    def _store(dst: oracle.Payload, src: oracle.Payload):
        dst.codes[:] = src.codes
        dst.scales[:] = src.scales
        dst.zps[:] = src.zps

    def quantize(self, x, e0, m, ref, bits, block):
        self._store(self.payload(ref, bits, block), oracle.quantize(x[e0:e0 + m], self.dtype, bits, block))

    def rs(self, ins, out, bits, block):
        p2 = oracle.rs_dequant_sum_requant([self.payload(r, bits, block) for r in ins])
        self._store(self.payload(out, bits, block), p2)

    def ag(self, ref, y, e0, m, bits, block):
        y[e0:e0 + m] = oracle.ag_dequant(self.payload(ref, bits, block), self.dtype)

    def new_output(self, x):
        return np.empty(x.shape[0], np.uint16)

    def sync(self):
        pass

    def close(self):
        for r, s in self.peers.items():
            if s is not self.shm:
                s.close()
        self.peers.clear()
        self.shm.close()
        self.shm.unlink()
