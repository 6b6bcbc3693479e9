"""The CPU oracle over every token row of a full-size workload, on all host
cores (test infrastructure).  Token-row slices of every rank are independent
all-reduces (each block depends only on the same block of every rank), so a
spawned pool runs the unmodified oracle on row slices and the slices of the
output and of every payload are concatenated in row order."""
import math
import multiprocessing as mp
import os

import numpy as np

import oracle


def _slice_allreduce(args):
    xs, dtype, bits, block = args
    y, p1, p2 = oracle.allreduce(list(xs), dtype, bits, block)
    return y, [(p.codes, p.scales, p.zps) for p in p1], (p2.codes, p2.scales, p2.zps)


def allreduce_all_rows(xs, T, H, dtype, bits, block, procs=None):
    """xs: P x (T*H) uint16.  Returns (y, [(codes, scales, zps)] * P, (codes, scales, zps))."""
    P = xs.shape[0]
    g = (P * block) // math.gcd(H, P * block)      # rows per slice stay whole P-block groups
    procs = procs or len(os.sched_getaffinity(0))
    nslices = max(1, min(procs * 2, T // g))
    cuts = [(T // g) * i // nslices * g for i in range(nslices)] + [T]
    jobs = [(np.ascontiguousarray(xs[:, cuts[i] * H:cuts[i + 1] * H]), dtype, bits, block)
            for i in range(nslices) if cuts[i + 1] > cuts[i]]
    with mp.get_context("spawn").Pool(min(procs, len(jobs))) as pool:
        parts = pool.map(_slice_allreduce, jobs)
    y = np.concatenate([p[0] for p in parts])
    p1 = [tuple(np.concatenate([p[1][r][f] for p in parts]) for f in range(3)) for r in range(P)]
    p2 = tuple(np.concatenate([p[2][f] for p in parts]) for f in range(3))
    return y, p1, p2
