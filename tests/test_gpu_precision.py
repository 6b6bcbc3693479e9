"""GPU parity of the per-step precision all-reduce (fc_quantized_allreduce_ex,
Fig. 5 right): every combination of reduce-scatter and all-gather widths in
{4, 8, 16} against the oracle's fco_allreduce_ex, bit for bit, including the
payloads of the quantized steps."""
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from bit_quantized_all_block_b200 import synth
from tests.gpu_util import assert_payload_equal, assert_y_equal, to_dev

pytestmark = pytest.mark.gpu

WIDTHS = [4, 8, 16]


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("b1", WIDTHS)
@pytest.mark.parametrize("b2", WIDTHS)
@pytest.mark.parametrize("P,block", [(2, 32), (4, 128), (8, 128), (4, 1024), (8, 4096)])
def test_precision_combinations(dtype, b1, b2, P, block):
    m = (3 * 4096) // (P * block) + 3
    n = P * block * m
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=block + P + b1 + 3 * b2)
    y_ref, p1_ref, p2_ref = oracle.allreduce_ex(list(xs), dtype, b1, b2, block)
    xd = to_dev(xs, dtype)
    s1 = [fc.QBuf.empty(n, b1, block) for _ in range(P)] if b1 != 16 else None
    s2 = fc.QBuf.empty(n, b2, block) if b2 != 16 else None
    y = fc.fc_quantized_allreduce_ex(xd, b1, b2, block, step1=s1, step2=s2)
    torch.cuda.synchronize()
    assert_y_equal(y, y_ref, f"y ({b1},{b2})")
    if s1 is not None:
        for r in range(P):
            assert_payload_equal(s1[r], p1_ref[r], f"step1[{r}]")
    if s2 is not None:
        assert_payload_equal(s2, p2_ref, "step2")
    y2 = fc.fc_quantized_allreduce_ex(xd, b1, b2, block)      # without payloads
    torch.cuda.synchronize()
    assert_y_equal(y2, y_ref, "y without payloads")


def test_precision_validation():
    xd = to_dev(synth.uniform_partials(3, 3 * 128 * 4, oracle.FP16, seed=1), oracle.FP16)
    with pytest.raises(fc.FCError) as e:
        fc.fc_quantized_allreduce_ex(xd, 8, 4, 128)          # mixed widths: P = 2, 4, 8 only
    assert e.value.status == fc.FC_ERR_UNSUPPORTED
    xd2 = xd[:2]
    with pytest.raises(fc.FCError) as e:
        fc.fc_quantized_allreduce_ex(xd2, 16, 8, 128, step1=[fc.QBuf.empty(xd2[0].numel(), 8, 128)] * 2)
    assert e.value.status == fc.FC_ERR_INVALID_ARG
    with pytest.raises(fc.FCError) as e:
        fc.fc_quantized_allreduce_ex(xd2, 8, 12, 128)
    assert e.value.status == fc.FC_ERR_INVALID_ARG
