"""The two-step quantized all-reduce across P GPUs, one process per GPU.

Flash Communication (sciencestack.ai/paper/2412.04964): in tensor-parallel
inference every rank holds a partial sum; the ranks quantize it, reduce-scatter
the low-bit payloads (each rank owns one chunk: it dequantizes that chunk from
every rank, sums in rank order and requantizes) and all-gather the owners'
payloads (TL;DR; Fig. 3; Fig. 5 right).  Here each rank is a process with its
own GPU, and "sending" a payload is the receiver's kernel reading it from the
sender's memory through a peer mapping (NVLink loads on a multi-GPU node).

Per call, rank r of P, n elements, chunk c = elements [c*m, (c+1)*m), m = n/P:

  1. quantize:        x_r[chunk c] -> S1_r[c]            for every c  (own memory)
  2. reduce-scatter:  S2_r = RS(S1_0[r], ..., S1_{P-1}[r])  (reads every peer)
  3. all-gather:      y[chunk c] = dequant(S2_c)         for every c  (reads owner c)

S1_r[c] and S2_r live in rank r's arena (`Layout`), each part 256-byte aligned.
After steps 1 and 2 every rank waits for its own stream and then for all
ranks (a host barrier), so a read never sees a payload before it is complete,
and no payload is rewritten while a peer may still read it: the next call's
step 1 (which rewrites S1) follows the barrier that ends every step 2, and its
step 2 (which rewrites S2) follows the barrier that every rank reaches only
after finishing step 3.  No kernel waits on another rank, so ranks that share
one GPU are valid too.

The arithmetic is that of one GPU's fused kernel, so the result is
bit-identical to `fc_quantized_allreduce` on the P partials.

The device operations come from an `ops` object (`CudaOps`: the library's
kernels, buffers in GPU memory, peers mapped with fc_ipc_open).

With one_kernel=True (one GPU per rank) each call is instead a single launch
of fc_p2p_allreduce: the same three steps inside one cooperative kernel per
rank, the ranks synchronised by counters in their arenas (system-scope
atomics and acquire loads through the peer mappings, bounded waits) instead
of host barriers; the kernel's payload and counter tables are built once, at
construction, since they depend only on the arenas.  Kernels of different
ranks then wait on each other, so this mode refuses ranks that share a GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import (P2PTables, PeerQBuf, fc_ag_dequant, fc_ipc_close, fc_ipc_export, fc_ipc_open, fc_p2p_allreduce,
               fc_payload_sizes, fc_quantize, fc_rs_dequant_sum_requant)

ALIGN = 256


def _align(v: int) -> int:
    return (v + ALIGN - 1) // ALIGN * ALIGN


@dataclass(frozen=True)
class PayloadRef:
    """A payload of `n` elements in rank `holder`'s arena (byte offsets)."""
    holder: int
    codes: int
    scales: int
    zps: int
    n: int


class Layout:
    """Byte offsets of every payload inside one rank's arena (the same on every rank)."""

    def __init__(self, n: int, P: int, bits: int, block: int):
        if P < 1 or n % (P * block) != 0:
            raise ValueError("n must be a multiple of P * block")
        self.n, self.P, self.bits, self.block = n, P, bits, block
        self.m = m = n // P
        cb, nb = fc_payload_sizes(m, bits, block)
        off = 0

        def take(nbytes: int) -> int:
            nonlocal off
            o = off
            off = _align(off + nbytes)
            return o

        self._step1 = [(take(cb), take(4 * nb), take(nb)) for _ in range(P)]
        self._step2 = (take(cb), take(4 * nb), take(nb))
        self.counters = take(8)          # phase-1 and phase-2 counters of the one-kernel mode (uint32 each)
        self.nbytes = off

    def step1(self, holder: int, c: int) -> PayloadRef:
        """Rank `holder`'s step-1 payload of chunk c."""
        return PayloadRef(holder, *self._step1[c], self.m)

    def step2(self, owner: int) -> PayloadRef:
        """The step-2 payload of chunk `owner`, held by its owner."""
        return PayloadRef(owner, *self._step2, self.m)


def ranks_share_a_device(device_ids) -> bool:
    """Whether two ranks report the same GPU (their one-kernel calls would wait
    on each other on one device, which nothing guarantees to make progress)."""
    return len(set(device_ids)) != len(device_ids)


def schedule(rank: int, layout: Layout):
    """The three steps of one call on `rank`, as data: (quantize targets per
    chunk, (RS inputs, RS output), all-gather sources per chunk)."""
    P = layout.P
    quantize = [layout.step1(rank, c) for c in range(P)]
    rs = ([layout.step1(r, rank) for r in range(P)], layout.step2(rank))
    ag = [layout.step2(c) for c in range(P)]
    return quantize, rs, ag


class CudaOps:
    """Device side on CUDA: the arena is a uint8 tensor on this rank's GPU,
    peers' arenas are mapped with fc_ipc_open, steps run the library's kernels
    on the current stream."""

    def __init__(self, device=None):
        import torch
        self.torch = torch
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.arena = None
        self.base = {}
        self.opened = []

    def alloc(self, nbytes: int):
        # zeroed: the one-kernel mode's counters start at 0
        self.arena = self.torch.zeros(max(nbytes, ALIGN), dtype=self.torch.uint8, device=self.device)

    def device_id(self) -> str:
        return str(self.torch.cuda.get_device_properties(self.device).uuid)

    def export(self):
        return fc_ipc_export(self.arena.data_ptr())

    def attach(self, rank: int, exported: list):
        for r, (handle, off) in enumerate(exported):
            if r == rank:
                self.base[r] = self.arena.data_ptr()
            else:
                b = fc_ipc_open(handle)
                self.opened.append(b)
                self.base[r] = b + off

    def qbuf(self, ref: PayloadRef, bits: int, block: int) -> PeerQBuf:
        b = self.base[ref.holder]
        return PeerQBuf(b + ref.codes, b + ref.scales, b + ref.zps, ref.n, bits, block)

    def quantize(self, x, e0: int, m: int, ref: PayloadRef, bits: int, block: int):
        fc_quantize(x[e0:e0 + m], bits, block, out=self.qbuf(ref, bits, block))

    def rs(self, ins, out: PayloadRef, bits: int, block: int):
        fc_rs_dequant_sum_requant([self.qbuf(r, bits, block) for r in ins], bits, block,
                                  out=self.qbuf(out, bits, block))

    def ag(self, ref: PayloadRef, y, e0: int, m: int, bits: int, block: int):
        fc_ag_dequant(self.qbuf(ref, bits, block), y.dtype, y=y[e0:e0 + m])

    def new_output(self, x):
        return x.new_empty(x.shape[0])

    def sync(self):
        self.torch.cuda.current_stream(self.device).synchronize()

    def close(self):
        self.sync()
        for b in self.opened:
            fc_ipc_close(b)
        self.opened.clear()


class QuantizedAllReduce:
    """All-reduce of n fp16/bf16 elements across the ranks of a process group.

    Collective constructor (every rank, same arguments): allocates this rank's
    arena, exchanges the peer mappings.  Calling the object on this rank's
    partial x (n elements, flat) writes the all-reduced result to y (default: a
    new tensor) and returns it; every rank receives the same bits.

    Failures: the host barriers between the steps are monitored with `timeout`
    seconds; if a rank fails or leaves, the others' call raises RuntimeError
    within that time (naming the missing rank) instead of blocking.  After such
    an error the object is unusable; every rank must create a new one."""

    def __init__(self, n: int, bits: int, block: int, group=None, ops=None, one_kernel: bool = False,
                 timeout: float = 60.0):
        import datetime

        import torch.distributed as dist
        self.dist = dist
        # a rank that fails or leaves makes the others' next barrier raise after
        # `timeout` seconds (naming the missing rank) instead of waiting for good
        self.timeout = datetime.timedelta(seconds=timeout)
        self.group = group if group is not None else dist.group.WORLD
        self.rank = dist.get_rank(self.group)
        self.P = dist.get_world_size(self.group)
        if self.P > 8:
            raise ValueError("at most 8 ranks")
        backend = dist.get_backend(self.group)
        # host barriers and the handle exchange run on a CPU group
        self.host = self.group if backend == "gloo" else dist.new_group(
            ranks=dist.get_process_group_ranks(self.group), backend="gloo", timeout=self.timeout)
        self.bits, self.block = bits, block
        self.layout = Layout(n, self.P, bits, block)
        self.ops = ops if ops is not None else CudaOps()
        self.ops.alloc(self.layout.nbytes)
        exported = [None] * self.P
        dist.all_gather_object(exported, self.ops.export(), group=self.host)
        self.one_kernel = one_kernel
        if one_kernel:
            ids = [None] * self.P
            dist.all_gather_object(ids, self.ops.device_id(), group=self.host)
            if ranks_share_a_device(ids):
                raise ValueError("one_kernel needs one GPU per rank: the ranks' kernels wait on each other")
            self.status = self.ops.torch.zeros(1, dtype=self.ops.torch.int32, device=self.ops.device)
        self.ops.attach(self.rank, exported)
        self.plan = schedule(self.rank, self.layout)
        if one_kernel:      # every call passes the same payload and counter addresses: marshal them once
            L, P = self.layout, self.P
            self.tables = P2PTables(
                [self.ops.qbuf(L.step1(p, c), bits, block) for p in range(P) for c in range(P)],
                [self.ops.qbuf(L.step2(c), bits, block) for c in range(P)],
                [self.ops.base[p] + L.counters for p in range(P)],
                [self.ops.base[p] + L.counters + 4 for p in range(P)])
        self.barrier()      # every mapping is in place (and every counter zero) before the first read

    def barrier(self):
        self.ops.sync()
        self.dist.monitored_barrier(group=self.host, timeout=self.timeout, wait_all_ranks=True)

    def __call__(self, x, y=None):
        L, b, B = self.layout, self.bits, self.block
        x = x.reshape(-1)
        if x.shape[0] != L.n:
            raise ValueError(f"expected {L.n} elements, got {x.shape[0]}")
        if y is None:
            y = self.ops.new_output(x)
        if self.one_kernel:
            return self._one_kernel_call(x, y)
        quantize, (ins, out), ag = self.plan
        for c, ref in enumerate(quantize):
            self.ops.quantize(x, c * L.m, L.m, ref, b, B)
        self.barrier()
        self.ops.rs(ins, out, b, B)
        self.barrier()
        for c, ref in enumerate(ag):
            self.ops.ag(ref, y, c * L.m, L.m, b, B)
        return y

    def _one_kernel_call(self, x, y):
        # epoch 0: the kernel counts its calls on the counters themselves, so a
        # call captured in a CUDA graph can be replayed
        fc_p2p_allreduce(self.rank, x, y, self.bits, self.block, None, None, None, None, 0, self.status,
                         tables=self.tables)
        return y

    def last_status(self) -> int:
        """One-kernel mode: 0, or 1 if a wait of the last call gave up (synchronizes)."""
        return int(self.status.item()) if self.one_kernel else 0

    def close(self):
        """Unmap the peers' arenas (collective: every rank, after its last call)."""
        self.barrier()
        self.ops.close()
