"""PreparedAllReduce: the fused all-reduce with its arguments marshalled once.

CPU: the argument checks happen at construction, before any CUDA call.
GPU: every call on the same buffers gives the oracle's result for the buffers'
current contents (inputs rewritten in place between calls), with and without
payloads, with per-step widths, on a fixed side stream, and equal to the
regular call."""
import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from bit_quantized_all_block_b200 import synth


def test_arguments_are_checked_at_construction():
    x = [torch.zeros(4096, dtype=torch.float16) for _ in range(2)]
    y = torch.zeros(4096, dtype=torch.float16)
    with pytest.raises(ValueError):
        fc.PreparedAllReduce([x[0], torch.zeros(2048, dtype=torch.float16)], 8, 8, 128, y=y)
    with pytest.raises(ValueError):
        fc.PreparedAllReduce([x[0], torch.zeros(4096, dtype=torch.bfloat16)], 8, 8, 128, y=y)
    with pytest.raises(ValueError):       # pageable CPU memory is not something a kernel can read
        fc.PreparedAllReduce(x, 8, 8, 128, y=y)
    with pytest.raises(TypeError):
        fc.PreparedAllReduce([torch.zeros(4096, dtype=torch.float32)] * 2, 8, 8, 128, y=y)


class _FakeEntry:
    """Stands in for the C entry point: records the stream argument of each call."""

    def __init__(self):
        self.streams = []

    def __call__(self, *args):
        self.streams.append(args[-1])
        return fc.FC_OK


def _prepared_without_device(fixed):
    p = fc.PreparedAllReduce.__new__(fc.PreparedAllReduce)
    p._args, p.y, p._stream, p._fn = (), None, fixed, _FakeEntry()
    return p


class _Stream:
    def __init__(self, handle):
        self.cuda_stream = handle


def test_a_fixed_stream_with_handle_zero_is_used(monkeypatch):
    """The legacy default stream has handle 0: fixing it must not fall back to the current stream."""
    import ctypes

    def no_current_stream(stream):
        if stream is None:
            raise AssertionError("the current stream was consulted although a stream was fixed")
        return ctypes.c_void_p(stream.cuda_stream)

    monkeypatch.setattr(fc, "_stream", no_current_stream)
    p = _prepared_without_device(ctypes.c_void_p(0))
    p()
    p(stream=_Stream(0x1234))                     # a per-call stream still overrides the fixed one
    assert [s.value for s in p._fn.streams] == [None, 0x1234]


def test_without_a_fixed_stream_each_call_takes_the_current_one(monkeypatch):
    import ctypes
    seen = []

    def current(stream):
        seen.append(stream)
        return ctypes.c_void_p(0x99 if stream is None else stream.cuda_stream)

    monkeypatch.setattr(fc, "_stream", current)
    p = _prepared_without_device(None)
    p()
    p()
    assert seen == [None, None] and [s.value for s in p._fn.streams] == [0x99, 0x99]


def _dev(xs_u16, dtype):
    t = torch.float16 if dtype == oracle.FP16 else torch.bfloat16
    return [torch.from_numpy(x.view(np.int16).copy()).view(t).cuda() for x in xs_u16]


def _host(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("bits", [8, 4])
def test_repeated_calls_follow_the_buffer_contents(dtype, bits):
    P, block, T, H = 4, 128, 8, 8192          # the decode-shaped message
    xs = _dev(synth.partials(P, T, H, dtype, 0.0, 1.0, seed=90), dtype)
    s1 = [fc.QBuf.empty(T * H, bits, block) for _ in range(P)]
    s2 = fc.QBuf.empty(T * H, bits, block)
    call = fc.PreparedAllReduce(xs, bits, bits, block, step1=s1, step2=s2)
    for seed in (91, 92, 93):
        new = synth.partials(P, T, H, dtype, 0.05, 20.0, seed=seed)
        for x, h in zip(xs, _dev(new, dtype)):
            x.copy_(h)                           # same storage, new contents
        y = call()
        torch.cuda.synchronize()
        y_ref, p1, p2 = oracle.allreduce(list(new), dtype, bits, block)
        assert np.array_equal(_host(y), y_ref), f"seed {seed}: output differs"
        for q, p in zip(s1 + [s2], p1 + [p2]):
            assert np.array_equal(q.codes.cpu().numpy(), p.codes)
            assert np.array_equal(q.scales.cpu().numpy().view(np.uint32), p.scales.view(np.uint32))
            assert np.array_equal(q.zps.cpu().numpy(), p.zps)


@pytest.mark.gpu
def test_per_step_widths_and_a_side_stream_match_the_regular_call():
    P, block, T, H, dtype = 8, 256, 16, 4096, oracle.BF16
    xs = _dev(synth.partials(P, T, H, dtype, 0.001, 50.0, seed=94), dtype)
    torch.cuda.synchronize()                     # the inputs were written on the default stream
    side = torch.cuda.Stream()
    call = fc.PreparedAllReduce(xs, 8, 4, block, stream=side)
    with torch.cuda.stream(side):
        y = call()
    side.synchronize()
    y_reg = fc.fc_quantized_allreduce_ex(xs, 8, 4, block)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_reg.view(torch.int16))
    y_ref = oracle.allreduce_ex([_host(x) for x in xs], dtype, 8, 4, block)[0]
    assert np.array_equal(_host(y), y_ref)


@pytest.mark.gpu
def test_page_locked_host_buffers():
    """The prepared call on page-locked host inputs and output (the kernels read
    and write host memory directly), inputs rewritten in place between calls."""
    P, block, T, H, dtype = 4, 128, 8, 8192, oracle.FP16
    xs = [torch.empty(T * H, dtype=torch.float16).pin_memory() for _ in range(P)]
    y = torch.empty(T * H, dtype=torch.float16).pin_memory()
    call = fc.PreparedAllReduce(xs, 8, 8, block, y=y)
    for seed in (95, 96):
        new = synth.partials(P, T, H, dtype, 0.0, 1.0, seed=seed)
        for x, h in zip(xs, new):
            x.copy_(torch.from_numpy(h.view(np.int16).copy()).view(torch.float16))
        call()
        torch.cuda.synchronize()
        y_ref = oracle.allreduce(list(new), dtype, 8, block)[0]
        assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16), y_ref), f"seed {seed}"


def test_p2p_tables_keep_their_buffers_alive():
    """The tables hold raw addresses, so they hold the payload and counter tensors too:
    dropping the caller's references must not free memory the tables point into."""
    import gc
    import weakref

    class Buf:                                  # stands in for a payload with tensors
        def __init__(self, base):
            self.base = base

        def struct(self):
            return fc.fc_qbuf(self.base, self.base + 256, self.base + 512)

    P = 2
    s1 = [Buf(0x1000 * (i + 1)) for i in range(P * P)]
    s2 = [Buf(0x9000 * (i + 1)) for i in range(P)]
    refs = [weakref.ref(b) for b in s1 + s2]
    tables = fc.P2PTables(s1, s2, [0x100, 0x104], [0x108, 0x10C])
    del s1, s2
    gc.collect()
    assert all(r() is not None for r in refs)
    assert [q.codes for q in tables.args[0]] == [0x1000 * (i + 1) for i in range(P * P)]
    del tables
    gc.collect()
    assert all(r() is None for r in refs)
