"""The CPU baseline on every host core: token-row slices of every rank are
independent all-reduces, so the oracle run as a team of spawned processes
(one per slice) must give the oracle's output for the whole sample, bit for
bit, with slices that keep n a multiple of P x block."""
import numpy as np

import bench
import oracle
from bit_quantized_all_block_b200 import synth


def test_team_equals_one_process_run():
    w = bench.WORKLOADS["p4_fp16_8192x8192_int8_b128"]
    xs = synth.workload_partials(w, rows=24)
    times, y, procs = bench.oracle_team(w, xs, 24, 2, 3)
    y_ref, _, _ = oracle.allreduce(list(xs), w.dtype, w.bits, w.block)
    assert procs == 3 and len(times) == 2 and all(t > 0 for t in times)
    assert np.array_equal(y, y_ref)


def test_team_slices_respect_the_chunk_granularity():
    # P = 8, H = 4096, block 4096: a slice must hold a multiple of 8 rows
    w = bench.WORKLOADS["p8_bf16_16384x4096_int4_b4096"]
    xs = synth.workload_partials(w, rows=21)
    times, y, procs = bench.oracle_team(w, xs, 21, 1, 4)
    assert procs == 2                      # 21 rows -> 16 usable rows -> two slices of 8
    y_ref, _, _ = oracle.allreduce([x[: 16 * w.H] for x in xs], w.dtype, w.bits, w.block)
    assert np.array_equal(y, y_ref)
