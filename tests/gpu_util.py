"""Helpers shared by the GPU tests: host<->device conversion and comparison
of library results with the oracle (test infrastructure)."""
import numpy as np
import torch

import bit_quantized_all_block_b200 as fc
import oracle


def tdtype(dtype):
    return torch.float16 if dtype == oracle.FP16 else torch.bfloat16


def to_dev(xs_u16, dtype):
    """P x n uint16 host array -> list of P contiguous CUDA tensors."""
    xs_u16 = np.ascontiguousarray(xs_u16)
    return [torch.from_numpy(x.view(np.int16).copy()).view(tdtype(dtype)).cuda() for x in xs_u16]


def host_u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def assert_payload_equal(q: fc.QBuf, p: oracle.Payload, what=""):
    codes = q.codes.cpu().numpy()
    scales = q.scales.cpu().numpy()
    zps = q.zps.cpu().numpy()
    assert np.array_equal(codes, p.codes), f"{what}: codes differ at {np.nonzero(codes != p.codes)[0][:8]}"
    assert np.array_equal(scales.view(np.uint32), p.scales.view(np.uint32)), f"{what}: scales differ"
    assert np.array_equal(zps, p.zps), f"{what}: zero-points differ"


def assert_y_equal(y, y_ref, what=""):
    got = host_u16(y)
    bad = np.nonzero(got != y_ref)[0]
    assert bad.size == 0, f"{what}: {bad.size} outputs differ, first at {bad[:8]}"


def run_fused(xs_dev, bits, block, with_payloads=True):
    P, n = len(xs_dev), xs_dev[0].numel()
    s1 = [fc.QBuf.empty(n, bits, block) for _ in range(P)] if with_payloads else None
    s2 = fc.QBuf.empty(n, bits, block) if with_payloads else None
    y = fc.fc_quantized_allreduce(xs_dev, bits, block, step1=s1, step2=s2)
    torch.cuda.synchronize()
    return y, s1, s2


def run_staged(xs_dev, bits, block):
    s1 = [fc.fc_quantize(x, bits, block) for x in xs_dev]
    s2 = fc.fc_rs_dequant_sum_requant(s1, bits, block)
    y = fc.fc_ag_dequant(s2, xs_dev[0].dtype)
    torch.cuda.synchronize()
    return y, s1, s2
