"""Seeded synthetic tensor-parallel partial sums (inputs only; no quantization here).

Stand-in for the o_proj / down_proj activation partials that Flash Communication
all-reduces across a TP=4 group (sciencestack.ai/paper/2412.04964, Fig. 1 and
Fig. 3; Fig. 4 uses LLaMA-3-8B activations on C4).  Neither trained weights nor
C4 are available, so the partials are drawn from a fixed recipe that keeps the
structure the method cares about: per-hidden-channel magnitudes that vary
log-normally, a few outlier channels much larger than the rest, and values that
are independent per rank while the channel structure is shared by all ranks.

Recipe (numpy Philox, seed 0 by default):
  1. from the stream Philox(seed): s_c ~ LogNormal(0, 0.5) for the H hidden
     channels (float64), then round(frac * H) outlier channels chosen without
     replacement, whose s_c is multiplied by ``outlier_factor``;
  2. for rank r = 0..P-1, from its own stream Philox(seed).jumped(r + 1):
     z_r ~ N(0, 1) of shape (T, H) drawn as float32 in row-major order, and
     x_r = z_r * float32(s_c) (float32 product, broadcast over tokens);
  3. x_r is rounded to fp16 or bf16 (torch .to(), round-to-nearest-even;
     identical to numpy's astype(float16) for fp16).
The function returns the raw 16-bit patterns so that the CPU oracle and the
GPU receive identical bytes.

This module is the only code shared by the oracle-side tests and the GPU
library's tests and benchmark; it holds none of the method's arithmetic.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

FP16 = 0
BF16 = 1


@dataclass(frozen=True)
class Workload:
    """One synthetic all-reduce problem: P partials of shape T x H."""

    name: str
    P: int
    T: int
    H: int
    dtype: int          # FP16 / BF16
    bits: int
    block: int
    outlier_frac: float
    outlier_factor: float
    seed: int = 0

    @property
    def n(self) -> int:
        return self.T * self.H

    def describe(self) -> str:
        dt = "fp16" if self.dtype == FP16 else "bf16"
        return (f"P={self.P} {dt} [{self.T}x{self.H}] INT{self.bits} block {self.block}, "
                f"N(0,1)*LogNormal(0,0.5) channel scales, "
                f"{self.outlier_frac * 100:g}% outlier channels x{self.outlier_factor:g}, Philox seed {self.seed}")


# The five workload families (small decode-like problem, LLaMA-3-70B-shaped
# prefill partials at INT8 and INT4, LLaMA-3-8B-shaped partials over the block
# sweep of Fig. 4, and the decode regime).
SMALL_P2 = Workload("p2_fp16_64x1024_int8_b128", 2, 64, 1024, FP16, 8, 128, 0.01, 20.0)
PREFILL_70B_INT8 = Workload("p4_fp16_8192x8192_int8_b128", 4, 8192, 8192, FP16, 8, 128, 0.001, 50.0)
PREFILL_70B_INT4 = Workload("p4_fp16_8192x8192_int4_b128", 4, 8192, 8192, FP16, 4, 128, 0.001, 50.0)
BLOCK_SWEEP_8B = tuple(
    Workload(f"p8_bf16_16384x4096_int4_b{b}", 8, 16384, 4096, BF16, 4, b, 0.001, 50.0)
    for b in (4096, 1024, 512, 256, 128))
DECODE_P4 = Workload("p4_fp16_8x8192_int8_b128", 4, 8, 8192, FP16, 8, 128, 0.0, 1.0)


def message_sweep(bits: int):
    """Decode-regime message sweep: 16 KB .. 1 GB of fp16 per rank at P=4
    (2^13 .. 2^29 elements, rows of 8192 hidden)."""
    return [Workload(f"p4_fp16_msg{2 << lg}B_int{bits}_b128", 4, (1 << lg) // 8192, 8192,
                     FP16, bits, 128, 0.0, 1.0) for lg in range(13, 30)]


def channel_scales(rng: np.random.Generator, H: int, frac: float, factor: float) -> np.ndarray:
    s_c = rng.lognormal(mean=0.0, sigma=0.5, size=H)
    k = int(round(frac * H))
    if k > 0:
        idx = rng.choice(H, size=k, replace=False)
        s_c[idx] *= factor
    return s_c


def _to_bits(x32: np.ndarray, dtype: int) -> np.ndarray:
    import torch  # host tensors only: torch's CPU conversions round to nearest even
    t = torch.from_numpy(np.ascontiguousarray(x32)).to(torch.float16 if dtype == FP16 else torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def partials(P: int, T: int, H: int, dtype: int, outlier_frac: float, outlier_factor: float,
             seed: int = 0, rows: int | None = None) -> np.ndarray:
    """P x (T*H) uint16 array of fp16/bf16 bit patterns.

    ``rows`` < T returns only the first ``rows`` tokens of every rank; since
    every rank draws from its own stream in row-major order, such a sample is
    exactly a prefix of the full workload."""
    rng = np.random.Generator(np.random.Philox(seed))
    s32 = channel_scales(rng, H, outlier_frac, outlier_factor).astype(np.float32)
    R = T if rows is None else min(rows, T)
    out = np.empty((P, R * H), dtype=np.uint16)

    def one_rank(r):
        rng_r = np.random.Generator(np.random.Philox(seed).jumped(r + 1))
        z = rng_r.standard_normal((R, H), dtype=np.float32)
        out[r] = _to_bits(z * s32[None, :], dtype).ravel()

    # ranks draw from independent streams, so they can be generated concurrently
    with ThreadPoolExecutor(max_workers=min(P, os.cpu_count() or 1)) as ex:
        list(ex.map(one_rank, range(P)))
    return out


def workload_partials(w: Workload, rows: int | None = None) -> np.ndarray:
    return partials(w.P, w.T, w.H, w.dtype, w.outlier_frac, w.outlier_factor, w.seed, rows)


def uniform_partials(P: int, n: int, dtype: int, seed: int, lo: float = -1.0, hi: float = 1.0,
                     zero_frac: float = 0.0) -> np.ndarray:
    """Small random partials for parity tests: uniform values, optional exact zeros."""
    rng = np.random.Generator(np.random.Philox(seed))
    x = rng.uniform(lo, hi, size=(P, n)).astype(np.float32)
    if zero_frac > 0:
        x[rng.random((P, n)) < zero_frac] = 0.0
    return np.stack([_to_bits(x[r], dtype) for r in range(P)])
