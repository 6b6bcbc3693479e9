"""Host buffers through the C ABI: page-locked host memory passed by its
device address (fc_host_device_pointer) is read and written by the kernels
themselves over the bus.  Results must be the oracle's bits, for the fused
all-reduce and for the staged steps, including pointers inside a larger
page-locked allocation."""
import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from bit_quantized_all_block_b200 import synth
from tests.gpu_util import assert_payload_equal, tdtype

pytestmark = pytest.mark.gpu


def _pinned(a_u16, dtype, offset=0):
    """A page-locked CPU tensor holding a_u16, `offset` elements into a larger one."""
    buf = torch.empty(a_u16.size + offset + 64, dtype=tdtype(dtype)).pin_memory()
    t = buf[offset:offset + a_u16.size]
    t.copy_(torch.from_numpy(a_u16.view(np.int16).copy()).view(tdtype(dtype)))
    return t


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("offset", [0, 8, 16])     # 16-byte and 32-byte aligned interior pointers
def test_fused_allreduce_on_host_buffers(dtype, bits, offset):
    P, block = 4, 128
    n = P * block * 37
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=70 + bits + offset)
    y_ref, p1_ref, p2_ref = oracle.allreduce(list(xs), dtype, bits, block)
    xh = [_pinned(x, dtype, offset) for x in xs]
    yh = _pinned(np.zeros(n, np.uint16), dtype, offset)
    s1 = [fc.QBuf.empty(n, bits, block) for _ in range(P)]
    s2 = fc.QBuf.empty(n, bits, block)
    fc.fc_quantized_allreduce(xh, bits, block, y=yh, step1=s1, step2=s2)
    torch.cuda.synchronize()
    assert np.array_equal(yh.view(torch.int16).numpy().view(np.uint16), y_ref)
    for q, p in zip(s1 + [s2], p1_ref + [p2_ref]):
        assert_payload_equal(q, p, "payload")


def test_staged_steps_on_host_buffers():
    P, bits, block, dtype = 3, 8, 256, oracle.FP16
    n = P * block * 20
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=77)
    y_ref, _, _ = oracle.allreduce(list(xs), dtype, bits, block)
    xh = [_pinned(x, dtype) for x in xs]
    s1 = [fc.fc_quantize(x, bits, block) for x in xh]          # host input, payload on the GPU
    s2 = fc.fc_rs_dequant_sum_requant(s1, bits, block)
    yh = _pinned(np.zeros(n, np.uint16), dtype)
    fc.fc_ag_dequant(s2, tdtype(dtype), y=yh)                  # result straight into host memory
    torch.cuda.synchronize()
    assert np.array_equal(yh.view(torch.int16).numpy().view(np.uint16), y_ref)


def test_unpinned_host_memory_is_refused_before_any_launch():
    x = torch.zeros(4096, dtype=torch.float16)                 # pageable
    with pytest.raises(ValueError):
        fc.fc_quantized_allreduce([x, x.clone()], 8, 128, y=torch.empty(4096, dtype=torch.float16).pin_memory())
    with pytest.raises(fc.FCError):
        fc.fc_host_device_pointer(x.data_ptr())
