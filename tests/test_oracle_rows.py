"""The row-parallel oracle helper used by the full-size GPU tests gives the
one-process oracle's output and payloads bit for bit (row slices that keep
whole P-block groups, concatenated in order)."""
import numpy as np

import oracle
from bit_quantized_all_block_b200 import synth
from tests.oracle_rows import allreduce_all_rows


def test_row_slices_reproduce_the_whole_allreduce():
    for P, T, H, dt, bits, block in ((4, 40, 1024, oracle.FP16, 8, 128), (8, 24, 4096, oracle.BF16, 4, 4096)):
        xs = synth.partials(P, T, H, dt, 0.01, 20.0, seed=3)
        y, p1, p2 = allreduce_all_rows(xs, T, H, dt, bits, block, procs=3)
        y_ref, p1_ref, p2_ref = oracle.allreduce(list(xs), dt, bits, block)
        assert np.array_equal(y, y_ref)
        for (codes, scales, zps), ref in zip(p1 + [p2], p1_ref + [p2_ref]):
            assert np.array_equal(codes, ref.codes)
            assert np.array_equal(scales.view(np.uint32), ref.scales.view(np.uint32))
            assert np.array_equal(zps, ref.zps)
