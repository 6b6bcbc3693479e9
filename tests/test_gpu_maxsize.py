"""The largest message of the sweep: P = 4 fp16 partials of 2^29 elements
(1 GB) each, INT8 and INT4, blocks of 128, both payloads written -- the sizes
the message sweep times at its top end.  The oracle cannot run over the whole
tensor in test time, so sampled token rows are checked bit for bit: each block
lies inside one row, so any set of rows of all ranks is an all-reduce of its
own, and the oracle runs on just those rows.  The rows include the first and
last rows, the rows around every chunk boundary and random rows.  The staged
pipeline must equal the fused kernel over the whole tensor.  Inputs are drawn
on the device with the sweep's recipe (N(0,1) values times LogNormal(0, 0.5)
channel scales, seeded)."""
import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle

pytestmark = pytest.mark.gpu

P, H, BLOCK = 4, 8192, 128
N = 1 << 29
T = N // H


def _partials(seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    scale = torch.exp(torch.randn(H, device="cuda", generator=g) * 0.5)
    xs = []
    for _ in range(P):
        x = torch.randn(T, H, device="cuda", generator=g)
        x.mul_(scale)
        xs.append(x.half().reshape(-1))
        del x
    return xs


def _rows(seed):
    rng = np.random.default_rng(seed)
    edges = {0, 1, T - 2, T - 1}
    for c in range(1, P):
        edges |= {c * T // P - 1, c * T // P}
    return np.array(sorted(edges | set(rng.choice(T, size=24, replace=False).tolist())))


@pytest.mark.parametrize("bits", [8, 4])
def test_largest_message_sampled_rows_and_staged(bits):
    xs = _partials(900 + bits)
    s1 = [fc.QBuf.empty(N, bits, BLOCK) for _ in range(P)]
    s2 = fc.QBuf.empty(N, bits, BLOCK)
    y = fc.fc_quantized_allreduce(xs, bits, BLOCK, step1=s1, step2=s2)
    torch.cuda.synchronize()

    rows = _rows(bits)
    idx = torch.from_numpy(rows).cuda()
    xr = np.stack([x.view(T, H)[idx].reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16) for x in xs])
    y_ref, p1_ref, p2_ref = oracle.allreduce(list(xr), oracle.FP16, bits, BLOCK)
    got = y.view(T, H)[idx].reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)
    bad = np.nonzero(got != y_ref)[0]
    assert bad.size == 0, f"{bad.size} sampled outputs differ, first at {bad[:8]}"

    cb, nb = H * bits // 8, H // BLOCK          # code bytes and blocks per row
    for q, p in zip(s1 + [s2], p1_ref + [p2_ref]):
        assert np.array_equal(q.codes.view(T, cb)[idx].cpu().numpy().reshape(-1), p.codes)
        assert np.array_equal(q.scales.view(T, nb)[idx].cpu().numpy().reshape(-1).view(np.uint32),
                              p.scales.view(np.uint32))
        assert np.array_equal(q.zps.view(T, nb)[idx].cpu().numpy().reshape(-1), p.zps)
    del s1

    q1 = [fc.fc_quantize(x, bits, BLOCK) for x in xs]
    q2 = fc.fc_rs_dequant_sum_requant(q1, bits, BLOCK)
    del q1
    y_st = fc.fc_ag_dequant(q2, torch.float16)
    torch.cuda.synchronize()
    assert torch.equal(y_st.view(torch.int16), y.view(torch.int16))
    assert torch.equal(q2.codes, s2.codes) and torch.equal(q2.zps, s2.zps)
    assert torch.equal(q2.scales.view(torch.int32), s2.scales.view(torch.int32))
