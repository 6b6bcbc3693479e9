"""Oracle argument and input validation."""
import numpy as np
import pytest

import oracle


def xs(P, n):
    return [np.zeros(n, np.uint16) for _ in range(P)]


@pytest.mark.parametrize("P,n,bits,block", [
    (2, 256, 3, 128),      # bits not 4/8
    (2, 256, 8, 3),        # odd block
    (2, 256, 8, 0),        # empty block
    (2, 200, 8, 128),      # n not a multiple of block
    (4, 384, 8, 128),      # n not a multiple of P*block
])
def test_bad_shapes(P, n, bits, block):
    with pytest.raises(oracle.OracleError):
        oracle.allreduce(xs(P, n), oracle.FP16, bits, block)


def test_empty_input_is_a_no_op():
    y, p1, p2 = oracle.allreduce(xs(2, 0), oracle.FP16, 8, 128)
    assert y.size == 0 and p2.codes.size == 0


@pytest.mark.parametrize("bad", [0x7C00, 0xFC00, 0x7E00])   # +inf, -inf, nan
def test_non_finite_input_is_rejected(bad):
    x = xs(2, 256)
    x[1][5] = bad
    with pytest.raises(oracle.OracleError):
        oracle.allreduce(x, oracle.FP16, 8, 128)
