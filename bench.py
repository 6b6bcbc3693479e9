"""Benchmark of the fused two-step quantized all-reduce on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--variant fused|fused_nopayload|staged]

One step = one whole quantized all-reduce of the workload (step-1 quantize
of every rank, reduce-scatter dequant-sum-requant, all-gather dequant) over
one batch of seeded synthetic partials already resident in HBM.  Default
workload: P=4 ranks of fp16 [8192 x 8192] partials (LLaMA-3-70B-shaped
prefill o_proj partial sums), INT8 in both steps, block 128.  The metric is
GB/s of input consumed (P*N*2 bytes per step); the roofline object reports
the algorithmic bytes of the kernel against the measured HBM copy bandwidth.

The N > 1 launch (torchrun, one process per GPU) runs an independent replica
of the whole P-rank problem on every GPU -- the method's ranks are emulated
inside one GPU, so there is no data-path collective; NCCL carries only the
barrier and the max-over-ranks of the timings.  ``value`` is the aggregate
over all GPUs.  After the timed replicas the N > 1 line also carries a
``collective`` object: the P = N quantized all-reduce across the job's GPUs
against NCCL's fp16 all-reduce at three message sizes (``--no-collective``
leaves it out; ``--collective`` runs the full message sweep).

``--impl reference`` times the CPU oracle (the plain definition the kernels
are checked against) on a bounded sample of the same workload, on rank 0.

Before every timed region, untimed steps worth ``--ramp-ms`` (default 300 ms)
of device time are enqueued directly ahead of it, with no host
synchronisation in between, so that however few steps are timed they run at
the GPU's running clocks (starting the clock sampler leaves the GPU idle).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_quantized_all_block_b200 import synth  # noqa: E402

WORKLOADS = {w.name: w for w in (synth.SMALL_P2, synth.PREFILL_70B_INT8, synth.PREFILL_70B_INT4,
                                 *synth.BLOCK_SWEEP_8B, synth.DECODE_P4)}
DEFAULT_WORKLOAD = synth.PREFILL_70B_INT8.name
METRIC = "quantized all-reduce input GB/s and % of HBM roofline (1×B200)"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_THRESHOLD = 256 << 20     # steps moving less than ~2x L2 (126 MB) get a cold-L2 timing
FLUSH_BYTES = 512 << 20
# sources of the fused all-reduce kernel (the dominant kernel of the default bench)
KERNEL_SOURCES = [os.path.join(ROOT, "bit_quantized_all_block_b200", "csrc", f)
                  for f in ("fc_device.cuh", "fc_kernels.cuh", "fc_fused.cuh", "fc_launch_impl.cuh")]


def payload_bytes(w) -> int:
    """Wire bytes of one quantization of n elements: codes + fp32 scale + u8 zero-point."""
    return w.n * w.bits // 8 + 5 * (w.n // w.block)


def algorithmic_bytes(w, variant: str) -> int:
    e = 2
    w2 = payload_bytes(w)
    w1 = w.P * w2
    if variant == "fused":
        return w.P * w.n * e + w.n * e + w1 + w2
    if variant == "fused_nopayload":
        return w.P * w.n * e + w.n * e
    if variant == "staged":
        return w.P * w.n * e + 2 * w1 + 2 * w2 + w.n * e
    raise ValueError(variant)


def _code_only(text: str) -> str:
    """C++ source with comments removed and whitespace collapsed (comment edits
    do not change the compiled kernel, so they keep the recorded traffic valid)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        h.update(os.path.basename(p).encode())
        h.update(_code_only(open(p).read()).encode())
    return h.hexdigest()[:16]


def read_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def read_traffic(workload: str, variant: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", f"traffic_{variant}_{workload}.txt")
    try:
        kv = dict(line.split(":", 1) for line in open(p).read().splitlines() if ":" in line)
    except OSError:
        return None
    if kv.get("kernel_source_hash", "").strip() != source_hash():
        return None
    try:
        return int(kv["dram_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,clocks.mem")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons, power, mem = [], None, set(), [], []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            try:
                power.append(float(f[3]))
                if len(f) > 9:
                    mem.append(float(f[9]))
            except ValueError:
                pass
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None,
                "mem_mhz": statistics.median(mem) if mem else None}


def max_over_ranks(v: float, world: int, device="cuda") -> float:
    """Max of a per-rank timing over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_gpu: int, world: int, ms: float) -> float:
    """Whole-job GB/s: every GPU processes bytes_per_gpu in the max-over-ranks time ms."""
    return world * bytes_per_gpu / (ms * 1e-3) / 1e9


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---- the CPU oracle on every host core (the cpu_baseline leg and --impl reference) ----
# Blocks are independent, so a token-row slice of every rank is a complete
# all-reduce of its own: one spawned process per core runs the unmodified
# oracle on its slice.  All processes meet at a barrier before each run; a
# run's time is the latest finish minus the earliest start.

def _oracle_team_worker(idx, xs_slice, dtype, bits, block, runs, barrier, out_q):
    import oracle
    oracle.lib()
    for k in range(runs):
        barrier.wait(timeout=600)
        t0 = time.time()
        y, _, _ = oracle.allreduce(list(xs_slice), dtype, bits, block)
        t1 = time.time()
        out_q.put((idx, k, t0, t1, y if k == runs - 1 else None))


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_team(w, xs, rows: int, runs: int, procs: int):
    """Run the oracle on the first `rows` token rows of every rank, split over
    `procs` processes, `runs` times.  Returns (seconds per run, y of the last
    run, processes used)."""
    import math
    import multiprocessing as mp
    g = (w.P * w.block) // math.gcd(w.H, w.P * w.block)     # rows per slice stay a whole all-reduce
    rows -= rows % g
    procs = max(1, min(procs, rows // g))
    cuts = [(rows // g) * i // procs * g for i in range(procs + 1)]
    ctx = mp.get_context("spawn")
    barrier, q = ctx.Barrier(procs), ctx.Queue()
    team = [ctx.Process(target=_oracle_team_worker, daemon=True,
                        args=(i, np.ascontiguousarray(xs[:, cuts[i] * w.H: cuts[i + 1] * w.H]),
                              w.dtype, w.bits, w.block, runs, barrier, q)) for i in range(procs)]
    for p in team:
        p.start()
    import queue
    stamps = [[None] * procs for _ in range(runs)]
    ys = [None] * procs
    ok = False
    try:
        got, deadline = 0, time.time() + 900
        while got < procs * runs:
            try:
                i, k, t0, t1, y = q.get(timeout=1.0)
            except queue.Empty:
                if any(p.exitcode not in (None, 0) for p in team):
                    raise RuntimeError("an oracle process exited early")
                if time.time() > deadline:
                    raise TimeoutError("the oracle processes did not finish")
                continue
            got += 1
            stamps[k][i] = (t0, t1)
            if y is not None:
                ys[i] = y
        ok = True
    finally:
        for p in team:
            p.join(timeout=30 if ok else 0.1)
            if p.is_alive():
                p.kill()
    times = [max(t1 for _, t1 in st) - min(t0 for t0, _ in st) for st in stamps]
    return times, np.concatenate(ys), procs


def run_reference(args, w):
    """The CPU oracle, as it stands, on a bounded row sample per step (rank 0 only)."""
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    cores = host_cores()
    rows = min(w.T, args.ref_rows * cores)
    xs = synth.workload_partials(w, rows=rows)
    times, _, procs = oracle_team(w, xs, rows, args.warmup + args.steps, cores)
    dt = sum(times[args.warmup:]) / args.steps
    value = xs.size * 2 / dt / 1e9
    sample = (f"first {rows} of {w.T} token rows of every rank ({xs.size} input elements per step), "
              f"split over {procs} processes, one per host core")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "description": w.describe(), "sample": sample},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": procs, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model()},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_precision_sweep(args, w):
    """Per-step precision (Fig. 5 right of the page): every width pair on one
    GPU, timed like the main bench, with the MSE of each against the fp32 sum."""
    import torch

    import bit_quantized_all_block_b200 as fc

    torch.cuda.set_device(0)
    xs_host = synth.workload_partials(w)
    tdt = torch.float16 if w.dtype == synth.FP16 else torch.bfloat16
    xs = [torch.from_numpy(x.view(np.int16)).view(tdt).cuda() for x in xs_host]
    S = xs[0].float()
    for x in xs[1:]:
        S = S + x.float()                        # fp32, rank order
    S64 = S.double()
    y = torch.empty(w.n, dtype=tdt, device="cuda")
    for b1 in (16, 8, 4):
        for b2 in (16, 8, 4):
            s1 = [fc.QBuf.empty(w.n, b1, w.block) for _ in range(w.P)] if b1 != 16 else None
            s2 = fc.QBuf.empty(w.n, b2, w.block) if b2 != 16 else None

            def step():
                fc.fc_quantized_allreduce_ex(xs, b1, b2, w.block, y=y, step1=s1, step2=s2)

            for _ in range(args.warmup):
                step()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.steps):
                step()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
            err = y.double() - S64
            mse = float((err * err).mean())
            w1 = w.n * b1 // 8 + 5 * (w.n // w.block) if b1 != 16 else 0
            w2 = w.n * b2 // 8 + 5 * (w.n // w.block) if b2 != 16 else 0
            alg = w.P * w.n * 2 + w.n * 2 + w.P * w1 + w2
            print(json.dumps({
                "metric": METRIC, "mode": "precision_sweep", "workload": w.name,
                "bits_rs": b1, "bits_ag": b2, "us": round(ms * 1e3, 2),
                "input_gbs": round(w.P * w.n * 2 / (ms * 1e-3) / 1e9, 1),
                "achieved_gbs": round(alg / (ms * 1e-3) / 1e9, 1),
                "mse_vs_fp32_sum": mse, "rel_mse": mse / float((S64 * S64).mean()),
                "wire_bytes_per_rank": (w1 if b1 != 16 else w.n * 2) + (w2 if b2 != 16 else w.n * 2)}),
                flush=True)
            del s1, s2


def run_gemm(args):
    """The GEMM with the fused step-1 quantizer (tensor cores), on the o_proj
    shape of the 70B-shaped workload: one rank's partial of [8192 tokens x 8192
    hidden] over its K = 8192/4 = 2048 slice, INT8 blocks of --gemm-block
    (default 128).  Compared with cuBLAS for the same GEMM followed by the
    separate quantize kernel."""
    import torch

    import bit_quantized_all_block_b200 as fc

    torch.cuda.set_device(0)
    M, N, K = args.gemm_shape
    B = args.gemm_block
    g = torch.Generator().manual_seed(0)
    a = torch.randn(M, K, generator=g).bfloat16().cuda()
    w = (torch.randn(N, K, generator=g) / K ** 0.5).bfloat16().cuda()
    q = fc.QBuf.empty(M * N, 8, B)
    part = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    # The variants are timed in interleaved rounds (each round times every
    # variant once, K calls each) and each reports its median over the rounds:
    # under the 1 kW power cap a variant timed later in a process runs slower,
    # so timing them one after the other would favour whichever goes first.
    variants = {
        "fused": lambda: fc.fc_gemm_quantize(a, w, 8, B, out=q, status=status),
        "plain": lambda: fc.fc_gemm_quantize(a, w, 8, B, partial=part, status=status, quantize=False),
        "cublas": lambda: torch.matmul(a, w.t(), out=part),
        "quant": lambda: fc.fc_quantize(part.view(-1), 8, B, out=q),
    }
    rounds = {k: [] for k in variants}
    with ClockSampler(0) as clocks:
        for _ in range(5):
            for k, fn in variants.items():
                rounds[k].append(timed(fn))
    assert int(status[0].item()) == 0, "GEMM pipeline reported a timeout"
    ms_fused, ms_plain, ms_cublas, ms_quant = (statistics.median(rounds[k]) for k in ("fused", "plain", "cublas",
                                                                                        "quant"))
    # The whole tensor-parallel layer output for P ranks (the page's setting:
    # each rank's o_proj partial, then the all-reduce), three ways.
    P = args.gemm_ranks
    As = [torch.randn(M, K, generator=g).bfloat16().cuda() for _ in range(P)]
    Ws = [(torch.randn(N, K, generator=g) / K ** 0.5).bfloat16().cuda() for _ in range(P)]
    q1 = [fc.QBuf.empty(M * N, 8, B) for _ in range(P)]
    q2 = fc.QBuf.empty(M * N, 8, B)
    parts = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    yb = torch.empty(M * N, dtype=torch.bfloat16, device="cuda")

    def layer_fused():
        for r in range(P):
            fc.fc_gemm_quantize(As[r], Ws[r], 8, B, out=q1[r], status=status)
        fc.fc_rs_dequant_sum_requant(q1, 8, B, out=q2)
        fc.fc_ag_dequant(q2, torch.bfloat16, y=yb)

    def layer_unfused(b):
        for r in range(P):
            torch.matmul(As[r], Ws[r].t(), out=parts[r])
        fc.fc_quantized_allreduce_ex([p_.view(-1) for p_ in parts], b, b, B, y=yb)

    layers = {"fused": layer_fused, "q8": lambda: layer_unfused(8), "u16": lambda: layer_unfused(16)}
    lr = {k: [] for k in layers}
    for _ in range(3):
        for k, fn in layers.items():
            lr[k].append(timed(fn))
    ms_layer_fused, ms_layer_cublas_q8, ms_layer_cublas_16 = (statistics.median(lr[k]) for k in ("fused", "q8", "u16"))
    flops = 2.0 * M * N * K
    tflops = flops / (ms_fused * 1e-3) / 1e12
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        peak, kind = float(d["bf16_tflops"]), "measured burst"
    except (OSError, KeyError, ValueError):
        peak, kind = 1590.0, "fallback"
    print(json.dumps({
        "metric": "GEMM with fused step-1 quantization, TFLOP/s", "mode": "gemm", "value": round(tflops, 1),
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "us_per_call": round(ms_fused * 1e3, 2), "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"o_proj partial per rank M={M} N={N} K={K}, bf16, INT8 block {B}"},
        "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(tflops / peak, 4), "peak_kind": kind},
        "timing": "CUDA events around K back-to-back calls; the variants interleaved over 5 rounds, median",
        "compare_us": {"fused_gemm_quantize": round(ms_fused * 1e3, 2),
                       "our_gemm_partial_only": round(ms_plain * 1e3, 2),
                       "cublas_gemm": round(ms_cublas * 1e3, 2), "quantize_kernel": round(ms_quant * 1e3, 2),
                       "cublas_gemm_then_quantize": round((ms_cublas + ms_quant) * 1e3, 2)},
        "tp_layer_us": {"ranks": P,
                        "fused_gemm_quantize_then_rs_ag_int8": round(ms_layer_fused * 1e3, 2),
                        "cublas_gemms_then_fused_allreduce_int8": round(ms_layer_cublas_q8 * 1e3, 2),
                        "cublas_gemms_then_unquantized_allreduce": round(ms_layer_cublas_16 * 1e3, 2)},
        "gpu_launches": args.steps, "clocks": clocks.summary()}), flush=True)


def run_latency_sweep(args):
    """Decode regime: per-call latency of the fused all-reduce over the message
    sweep (16 KB .. 8 MB per rank, P=4, INT8 and INT4), then the decode-shaped
    message (8 tokens x 8192 hidden) at P=2 (INT8) and P=8 (INT4), measured two
    ways: back to back inside a CUDA graph (L2 warm: the kernel's own latency)
    and one call at a time after an L2 flush (cold)."""
    import torch

    import bit_quantized_all_block_b200 as fc

    torch.cuda.set_device(0)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    extra = [synth.Workload("p2_fp16_8x8192_int8_b128", 2, 8, 8192, synth.FP16, 8, 128, 0.0, 1.0),
             synth.Workload("p8_fp16_8x8192_int4_b128", 8, 8, 8192, synth.FP16, 4, 128, 0.0, 1.0)]
    for w in synth.message_sweep(8)[:10] + synth.message_sweep(4)[:10] + extra:
        bits = w.bits
        xs = [torch.from_numpy(x.view(np.int16)).view(torch.float16).cuda() for x in synth.workload_partials(w)]
        y = torch.empty(w.n, dtype=torch.float16, device="cuda")
        s1 = [fc.QBuf.empty(w.n, bits, w.block) for _ in range(w.P)]
        s2 = fc.QBuf.empty(w.n, bits, w.block)

        def step():
            fc.fc_quantized_allreduce(xs, bits, w.block, y=y, step1=s1, step2=s2)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(20):
                step()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        hot = e0.elapsed_time(e1) * 1e3 / 20
        pairs = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            step()
            b.record()
            pairs.append((a, b))
        torch.cuda.synchronize()
        cold = sorted(a.elapsed_time(b) * 1e3 for a, b in pairs)[len(pairs) // 2]
        print(json.dumps({"mode": "latency_sweep", "workload": w.name, "P": w.P, "bits": bits,
                          "bytes_per_rank": 2 * w.n, "us_graph_back_to_back": round(hot, 2),
                          "us_cold_l2_median": round(cold, 2),
                          "input_gbs_back_to_back": round(w.P * w.n * 2 / hot / 1e3, 1)}), flush=True)
        del g


def run_message_sweep(args):
    """The whole message sweep of the decode-to-prefill range: 16 KB .. 1 GB of
    fp16 per rank (2^13 .. 2^29 elements, P=4, INT8 and INT4, blocks of 128),
    the fused all-reduce with both payloads written.  Per size: back to back in
    a CUDA graph of 20 calls (L2 warm for the small sizes; beyond 32 MB per rank
    every call streams from HBM) and one call at a time after an L2 flush (cold,
    median).  Inputs are drawn on the device from a seeded generator with the
    synthetic recipe's shape (N(0,1) times per-channel log-normal scales); the
    largest point holds about 7.6 GB on the device."""
    import torch

    import bit_quantized_all_block_b200 as fc

    torch.cuda.set_device(0)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    peak, peak_kind = read_peak()
    gen = torch.Generator(device="cuda")
    for bits in (8, 4):
        for w in synth.message_sweep(bits):
            gen.manual_seed(1000 + w.T)
            scale = torch.exp(torch.randn(w.H, device="cuda", generator=gen) * 0.5)
            xs = [(torch.randn(w.T, w.H, device="cuda", generator=gen) * scale).half().reshape(-1)
                  for _ in range(w.P)]
            y = torch.empty(w.n, dtype=torch.float16, device="cuda")
            s1 = [fc.QBuf.empty(w.n, bits, w.block) for _ in range(w.P)]
            s2 = fc.QBuf.empty(w.n, bits, w.block)

            def step():
                fc.fc_quantized_allreduce(xs, bits, w.block, y=y, step1=s1, step2=s2)

            for _ in range(max(args.warmup, 3)):
                step()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(20):
                    step()
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            hot = e0.elapsed_time(e1) * 1e3 / 20
            pairs = []
            for _ in range(args.steps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                step()
                b.record()
                pairs.append((a, b))
            torch.cuda.synchronize()
            cold = sorted(a.elapsed_time(b) * 1e3 for a, b in pairs)[len(pairs) // 2]
            alg = algorithmic_bytes(w, "fused")
            print(json.dumps({"mode": "message_sweep", "workload": w.name, "bytes_per_rank": 2 * w.n,
                              "bits": bits, "us_back_to_back": round(hot, 2), "us_cold_l2_median": round(cold, 2),
                              "input_gbs_back_to_back": round(w.P * w.n * 2 / hot / 1e3, 1),
                              "achieved_gbs_back_to_back": round(alg / hot / 1e3, 1),
                              "frac_back_to_back": round(alg / hot / 1e3 / peak, 4), "peak_kind": peak_kind}),
                  flush=True)
            del g, xs, y, s1, s2
            torch.cuda.empty_cache()


# ---- the P-GPU exchange against NCCL (one process per GPU) ----------------------
# Flash Communication (sciencestack.ai/paper/2412.04964), Abstract and Fig. 1:
# the quantized two-step all-reduce against NCCL's fp16 ring all-reduce of the
# same partial, over the message range of decode to prefill.  The sweep logic
# is backend-neutral (`collective_sweep`); `CudaCollectiveEnv` is the GPU form
# run under torchrun, and the CPU tests drive the same function with gloo ranks.

COLLECTIVE_BLOCK = 128


def collective_points(P: int, block: int = COLLECTIVE_BLOCK, min_bytes: int = 16 << 10, max_bytes: int = 1 << 30):
    """(bits, elements per rank) of the sweep: fp16 messages of 16 KB .. 1 GB
    per rank in powers of two, INT8 then INT4, each rounded down to whole
    chunks of blocks (a multiple of P * block elements)."""
    sizes = []
    b = min_bytes
    while b <= max_bytes:
        n = (b // 2) // (P * block) * (P * block)
        if n > 0:
            sizes.append(n)
        b *= 2
    return [(bits, n) for bits in (8, 4) for n in sizes]


def wire_bytes_per_rank(P: int, n: int, bits: int, block: int) -> dict:
    """Bytes each rank receives per call: the quantized exchange pulls (P-1)/P
    of a payload in the reduce-scatter and again in the all-gather; NCCL's
    ring all-reduce moves 2 (P-1)/P of the fp16 message."""
    w2 = n * bits // 8 + 5 * (n // block)
    return {"quantized": 2 * (P - 1) * w2 // P, "nccl_fp16_ring": 2 * (P - 1) * 2 * n // P}


def collective_sweep(env, points, steps: int, warmup: int, emit, block: int = COLLECTIVE_BLOCK):
    """Time every form of the P-rank quantized all-reduce and the baseline
    all-reduce at each point; emit one dict per point (on rank 0).

    env supplies: rank, world, forms (names -> one_kernel flag; the one-kernel
    form only where each rank has its own GPU), partial(n) (this rank's seeded
    partial), expected(n, bits, block) (this rank's output of the one-GPU fused
    all-reduce of all P partials), allreduce(n, bits, block, one_kernel) (a
    QuantizedAllReduce), new_output(x), equal(a, b), baseline_buffer(x) and
    baseline(buf) (one fp16 all-reduce of the message), timed(fn) (elapsed ms
    of fn's work on this rank's device), barrier(), all_true(flag) and
    max_over_ranks(v).  Every rank runs the same collective calls in the same
    order."""
    P = env.world
    for bits, n in points:
        x = env.partial(n)
        want = env.expected(n, bits, block)
        us, exact, status = {}, {}, {}
        for name, one_kernel in env.forms.items():
            ar = env.allreduce(n, bits, block, one_kernel)
            y = env.new_output(x)
            ar(x, y)
            env.sync()
            exact[name] = env.all_true(env.equal(y, want))
            first = int(env.max_over_ranks(float(ar.last_status())))
            if first != 0:
                # a bounded wait gave up on some rank: the one-kernel form's
                # counters no longer match its epochs, so every later call would
                # give up too (after its wait limit); no rank times this form
                status[name], us[name] = first, None
                ar.close()
                continue
            for _ in range(warmup):
                ar(x, y)
            env.sync()
            env.barrier()

            def calls(ar=ar, y=y):
                for _ in range(steps):
                    ar(x, y)

            ms = env.timed(calls)
            status[name] = int(env.max_over_ranks(float(ar.last_status())))
            us[name] = env.max_over_ranks(ms / steps * 1e3)
            ar.close()
        buf = env.baseline_buffer(x)
        for _ in range(warmup):
            env.baseline(buf)
        env.sync()
        env.barrier()

        def base_calls():
            for _ in range(steps):
                env.baseline(buf)

        ms = env.timed(base_calls)
        us["nccl_fp16"] = env.max_over_ranks(ms / steps * 1e3)
        if env.rank == 0:
            emit({"mode": "collective", "P": P, "bits": bits, "block": block, "elements_per_rank": n,
                  "bytes_per_rank": 2 * n, "steps": steps, "warmup": warmup,
                  "us": {k: (round(v, 2) if v is not None else None) for k, v in us.items()},
                  "wire_bytes_per_rank": wire_bytes_per_rank(P, n, bits, block),
                  "speedup_vs_nccl_fp16": {k: round(us["nccl_fp16"] / v, 3) for k, v in us.items()
                                           if k != "nccl_fp16" and v is not None},
                  "bit_exact_vs_fused": exact, "wait_status": status,
                  "timing": env.timing_note})


class CudaCollectiveEnv:
    """The sweep on one GPU per rank: NCCL for the fp16 baseline, a gloo group
    for everything else between the ranks (the quantized all-reduce's host
    barriers and handle exchange, the sweep's barriers, flags and
    max-over-ranks), inputs drawn on the device (the synthetic recipe's shape:
    N(0,1) times per-channel log-normal scales over 8192 channels)."""

    timing_note = ("CUDA events on each rank's stream around K calls after W warm-up calls (the host-barrier "
                   "form's waits included), per call, max over ranks")

    def __init__(self, rank: int, world: int, local: int):
        import torch
        import torch.distributed as dist

        import bit_quantized_all_block_b200 as fc
        from bit_quantized_all_block_b200 import collective
        self.torch, self.dist, self.fc, self.collective = torch, dist, fc, collective
        self.rank, self.world = rank, world
        self.device = torch.device("cuda", local)
        self.stream = torch.cuda.current_stream()
        self.host = dist.new_group(backend="gloo", timeout=datetime.timedelta(seconds=120))
        ids = [None] * world
        dist.all_gather_object(ids, collective.CudaOps(self.device).device_id(), group=self.host)
        self.forms = {"host_barrier": False}
        if world in (2, 4, 8) and not collective.ranks_share_a_device(ids):
            self.forms["one_kernel"] = True

    def _draw(self, n: int, r: int):
        torch = self.torch
        H = 8192 if n % 8192 == 0 else n
        g = torch.Generator(device=self.device)
        g.manual_seed(7000 + n)
        scale = torch.exp(torch.randn(H, device=self.device, generator=g) * 0.5)
        g.manual_seed(7001 + n + 1000003 * r)
        return (torch.randn(n // H, H, device=self.device, generator=g) * scale).half().reshape(-1)

    def partial(self, n: int):
        return self._draw(n, self.rank)

    def expected(self, n: int, bits: int, block: int):
        xs = [self._draw(n, r) for r in range(self.world)]
        y = self.fc.fc_quantized_allreduce(xs, bits, block)
        del xs
        return y

    def allreduce(self, n, bits, block, one_kernel):
        return self.collective.QuantizedAllReduce(n, bits, block, group=self.host, one_kernel=one_kernel,
                                                  timeout=120.0)

    def new_output(self, x):
        return self.torch.empty_like(x)

    def equal(self, a, b) -> bool:
        return bool(self.torch.equal(a.view(self.torch.int16), b.view(self.torch.int16)))

    def baseline_buffer(self, x):
        return x.clone()

    def baseline(self, buf):
        self.dist.all_reduce(buf)

    def sync(self):
        self.torch.cuda.synchronize()

    # Coordination (barriers, flags, timings) runs on the gloo group: if one
    # rank's call fails, the others' next step ends with a gloo error after the
    # group's timeout instead of an NCCL operation left waiting, and NCCL runs
    # only the baseline all-reduce, which every rank reaches past the same gloo
    # steps.
    def barrier(self):
        self.dist.barrier(group=self.host)

    def timed(self, fn) -> float:
        torch = self.torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(self.stream)
        fn()
        b.record(self.stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    def all_true(self, flag: bool) -> bool:
        t = self.torch.tensor([1 if flag else 0], dtype=self.torch.int32)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MIN, group=self.host)
        return bool(t.item())

    def max_over_ranks(self, v: float) -> float:
        t = self.torch.tensor([v], dtype=self.torch.float64)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.host)
        return float(t.item())


def run_collective(args):
    """--collective: the sweep under torchrun, one process per GPU (2, 4 or 8
    for the one-kernel form); one JSON line per point on rank 0."""
    import torch
    import torch.distributed as dist

    world, rank, local = dist_setup(args)
    if world < 2:
        print(json.dumps({"mode": "collective", "unavailable": "needs 2 or more GPUs, one process per GPU "
                                                              "(torchrun --nproc-per-node N bench.py --collective)"}),
              flush=True)
        return
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    try:
        env = CudaCollectiveEnv(rank, world, local)
        max_bytes = args.collective_max_mb << 20
        collective_sweep(env, collective_points(world, max_bytes=max_bytes), args.steps, args.warmup,
                         lambda row: print(json.dumps(row), flush=True))
        torch.cuda.synchronize()
        dist.barrier()
    finally:
        dist.destroy_process_group()


# Message sizes of the collective object in the N > 1 line: the decode-shaped
# message (8 x 8192 fp16 per rank) at INT8, the prefill-shaped one
# (8192 x 8192 fp16 per rank) at INT8 and at INT4, blocks of 128.
LINE_COLLECTIVE_POINTS = [(8, 8 * 8192), (8, 8192 * 8192), (4, 8192 * 8192)]


def collective_in_line(args, world: int, rank: int, local: int):
    """N > 1: the P = N quantized all-reduce across the job's GPUs (one process
    per GPU, both forms) against NCCL's fp16 all-reduce at LINE_COLLECTIVE_POINTS,
    after the timed replicas.  Every rank runs it; rank 0 gets the object for its
    line.  A failure is reported in the object, not raised."""
    rows = []
    try:
        env = CudaCollectiveEnv(rank, world, local)
        collective_sweep(env, LINE_COLLECTIVE_POINTS, args.steps, args.warmup, rows.append)
        err = None
    except Exception as ex:                         # the replicas' line is printed all the same
        err = f"{type(ex).__name__}: {ex}"[:300]
    if rank != 0:
        return None
    return {"what": (f"the P = {world} quantized all-reduce across the job's GPUs (one process per GPU; peer "
                     f"payloads read through IPC mappings) against NCCL's fp16 all-reduce of the same partial, "
                     f"timed after the replicas"),
            "points": rows, "error": err}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--variant", default="fused",
                    help="fused | fused_nopayload | staged, or a comma-separated list (one JSON line each)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="token-row chunks of the pipelined host-buffer form of the e2e figure")
    ap.add_argument("--ref-rows", type=int, default=256,
                    help="token rows per rank in one reference (oracle) step")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="token rows per rank for the cpu_baseline sample (0 = the whole workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ramp-ms", type=float, default=300.0,
                    help="untimed device work (ms) enqueued directly before the timed region")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of replaying a CUDA graph of them")
    ap.add_argument("--gemm", action="store_true",
                    help="time the tensor-core GEMM with the fused step-1 quantizer (o_proj shape)")
    ap.add_argument("--gemm-shape", type=int, nargs=3, default=[8192, 8192, 2048], metavar=("M", "N", "K"))
    ap.add_argument("--gemm-ranks", type=int, default=4, help="ranks of the tensor-parallel layer comparison")
    ap.add_argument("--gemm-block", type=int, default=128, help="quantization block of --gemm (32, 64, 128 or 256)")
    ap.add_argument("--latency-sweep", action="store_true",
                    help="decode regime: per-call latency over the 16 KB .. 8 MB per rank message sweep")
    ap.add_argument("--message-sweep", action="store_true",
                    help="the fused all-reduce over 16 KB .. 1 GB per rank (P=4, INT8 and INT4), one line each")
    ap.add_argument("--collective", action="store_true",
                    help="under torchrun, one process per GPU: the P-GPU quantized all-reduce (host-barrier and "
                         "one-kernel forms) against NCCL's fp16 all-reduce over 16 KB .. 1 GB per rank")
    ap.add_argument("--collective-max-mb", type=int, default=1024,
                    help="largest message per rank of the --collective sweep (MB)")
    ap.add_argument("--no-collective", action="store_true",
                    help="N > 1: leave the P-GPU collective object out of the default line")
    ap.add_argument("--precision-sweep", action="store_true",
                    help="time the fused kernel for every (RS bits, AG bits) in {4,8,16}^2 on the "
                         "workload and report each variant's MSE (one JSON line per variant)")
    args = ap.parse_args()
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"
    for v in args.variant.split(","):
        assert v in ("fused", "fused_nopayload", "staged"), f"unknown variant {v}"
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.precision_sweep:
        return run_precision_sweep(args, w)
    if args.gemm:
        return run_gemm(args)
    if args.latency_sweep:
        return run_latency_sweep(args)
    if args.message_sweep:
        return run_message_sweep(args)
    if args.collective:
        return run_collective(args)

    import torch
    import torch.distributed as dist

    import bit_quantized_all_block_b200 as fc

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- inputs: seeded host generation, identical bytes on every rank -------
    xs_host = synth.workload_partials(w)
    tdt = torch.float16 if w.dtype == synth.FP16 else torch.bfloat16
    xs_pinned = [torch.from_numpy(x.view(np.int16)).view(tdt).pin_memory() for x in xs_host]
    xs = [x.cuda() for x in xs_pinned]
    y = torch.empty(w.n, dtype=tdt, device="cuda")
    s1 = [fc.QBuf.empty(w.n, w.bits, w.block) for _ in range(w.P)]
    s2 = fc.QBuf.empty(w.n, w.bits, w.block)
    stream = torch.cuda.current_stream()

    def staged_once(xs_, y_, s1_, s2_):
        for r in range(w.P):
            fc.fc_quantize(xs_[r], w.bits, w.block, out=s1_[r])
        fc.fc_rs_dequant_sum_requant(s1_, w.bits, w.block, out=s2_)
        fc.fc_ag_dequant(s2_, tdt, y=y_)

    def staged_timing(xs_, y_, s1_, s2_, small_, flush_):
        """K staged steps with events between the stages: (mean ms of each of the
        three stages, total ms of every step).  Like the fused steps, workloads
        larger than L2 are timed as one replay of a CUDA graph of the K steps
        (events recorded between the stages inside the graph), after replays
        worth --ramp-ms; smaller ones flush L2 before each step, launched one by
        one."""
        use_graph = not small_ and not args.no_graph
        marks = [[torch.cuda.Event(enable_timing=True, external=use_graph) for _ in range(4)]
                 for _ in range(args.steps)]

        def steps():
            for ev in marks:
                if small_:
                    flush_.zero_()
                ev[0].record()
                for r in range(w.P):
                    fc.fc_quantize(xs_[r], w.bits, w.block, out=s1_[r])
                ev[1].record()
                fc.fc_rs_dequant_sum_requant(s1_, w.bits, w.block, out=s2_)
                ev[2].record()
                fc.fc_ag_dequant(s2_, tdt, y=y_)
                ev[3].record()

        if use_graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                steps()
            torch.cuda.synchronize()
            g.replay()                          # one untimed replay, which also sizes the ramp
            torch.cuda.synchronize()
            t_replay = marks[0][0].elapsed_time(marks[-1][3])
            for _ in range(max(1, math.ceil(args.ramp_ms / max(t_replay, 1e-3)))):
                g.replay()
            g.replay()                          # the timed replay: the events hold its times
            torch.cuda.synchronize()
            del g
        else:
            steps()
            torch.cuda.synchronize()
        stage = [sum(m[i].elapsed_time(m[i + 1]) for m in marks) / args.steps for i in range(3)]
        return stage, [m[0].elapsed_time(m[3]) for m in marks]

    variants = args.variant.split(",")
    for vi, variant in enumerate(variants):
        def step(xs_=xs, y_=y):
            if variant == "fused":
                fc.fc_quantized_allreduce(xs_, w.bits, w.block, y=y_, step1=s1, step2=s2)
            elif variant == "fused_nopayload":
                fc.fc_quantized_allreduce(xs_, w.bits, w.block, y=y_)
            else:
                staged_once(xs_, y_, s1, s2)

        launches_per_step = 1 if variant.startswith("fused") else w.P + 2

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()

        # ---- timed region: K steps, events on the launching stream ---------------
        # Workloads larger than L2 run back to back (every step streams from HBM).
        # Smaller ones flush L2 with a 512 MB write before every step and time each
        # step with its own pair of events (the flush keeps the GPU busy while the
        # host enqueues the step, so no host gap falls inside the pair).
        step_bytes = algorithmic_bytes(w, variant)
        small = step_bytes < L2_FLUSH_THRESHOLD
        graph = None
        # per-step marks: recorded between the steps (inside the graph as event
        # record nodes), read after the timed replay for the per-step spread
        step_marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(args.steps + 1)]
        if not small and variant != "staged" and not args.no_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step_marks[0].record()
                for i in range(args.steps):
                    step()
                    step_marks[i + 1].record()
            torch.cuda.synchronize()
            graph.replay()                      # one untimed replay
            torch.cuda.synchronize()
        flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda") if small else None
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        # Clock ramp: starting the clock sampler leaves the GPU idle for a few
        # hundred ms, and its clocks drop.  Untimed work for at least --ramp-ms of
        # device time is therefore enqueued directly before the timed region,
        # with no host synchronisation between the two, so the timed steps run at
        # the GPU's running clocks however few they are.  The default 300 ms also
        # lets the power draw settle: the headline all-reduce ran 2 % faster and
        # steadier after 300 ms than after 100 ms, alternating on one GPU.
        def unit():
            if graph is not None:
                graph.replay()
            else:
                if small:
                    flush.zero_()
                step()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(stream)
        unit()
        eb.record(stream)
        torch.cuda.synchronize()
        n_ramp = max(1, math.ceil(args.ramp_ms / max(ea.elapsed_time(eb), 1e-3)))
        ramp_steps = n_ramp * (args.steps if graph is not None else 1)

        with ClockSampler(local) as clocks:
            barrier()
            torch.cuda.synchronize()
            for _ in range(n_ramp):
                unit()
            if variant == "staged":
                stage_ms, step_ms = staged_timing(xs, y, s1, s2, small, flush)
                ms = sum(stage_ms)
            elif not small:
                # the K steps are captured once in a CUDA graph and replayed, so
                # host launch gaps do not enter the device time
                ev0.record(stream)
                if graph is not None:
                    graph.replay()
                else:
                    step_marks[0].record(stream)
                    for i in range(args.steps):
                        step()
                        step_marks[i + 1].record(stream)
                ev1.record(stream)
                torch.cuda.synchronize()
                ms = ev0.elapsed_time(ev1) / args.steps
                step_ms = [step_marks[i].elapsed_time(step_marks[i + 1]) for i in range(args.steps)]
            else:
                pairs = []
                for _ in range(args.steps):
                    flush.zero_()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    step()
                    b.record(stream)
                    pairs.append((a, b))
                torch.cuda.synchronize()
                step_ms = [a.elapsed_time(b) for a, b in pairs]
                ms = sum(step_ms) / args.steps
            # the fused line also carries the staged pipeline's roofline, timed in
            # the same run on the same inputs (its own ramp, K steps)
            staged_extra = None
            if variant == "fused":
                if small:       # the graph form carries its own ramp
                    for _ in range(max(1, math.ceil(args.ramp_ms / max(ms * 3, 1e-3)))):
                        staged_once(xs, y, s1, s2)
                st_stage_ms, st_step_ms = staged_timing(xs, y, s1, s2, small, flush)
                staged_extra = (st_stage_ms, st_step_ms)
            barrier()
        ms = max_over_ranks(ms, world)
        ms_median = max_over_ranks(statistics.median(step_ms), world)
        ms_min = max_over_ranks(min(step_ms), world)

        # ---- end to end through the public API with host buffers -----------------
        # The same calls on the page-locked host inputs and a page-locked host
        # output: the kernels read the inputs from host memory and write the
        # result there themselves (zero-copy through the bus), so every step's
        # host->device and device->host traffic is inside the timed region.
        # The explicit-copy form (asynchronous copies of the inputs, the call on
        # device buffers, a copy of the result back) is timed beside it.
        y_host = torch.empty(w.n, dtype=tdt).pin_memory()

        def e2e_copies():
            for r in range(w.P):
                xs[r].copy_(xs_pinned[r], non_blocking=True)
            step()
            y_host.copy_(y, non_blocking=True)

        def e2e_zero_copy():
            step(xs_pinned, y_host)

        # Pipelined: token-row chunks (each an all-reduce of its own, every block
        # lying in one chunk) on three streams, so the H2D copy of chunk c + 1,
        # the fused call on chunk c and the D2H copy of chunk c - 1 overlap.
        unit = w.H * (w.P * w.block) // math.gcd(w.H, w.P * w.block)
        nchunks = min(args.e2e_chunks, w.n // unit) if variant.startswith("fused") else 0
        bounds = []
        if nchunks > 1:
            per = (w.n // unit // nchunks) * unit
            bounds = [(c * per, (c + 1) * per if c + 1 < nchunks else w.n) for c in range(nchunks)]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def qslice(q, e0, e1):
            return fc.QBuf(q.codes[e0 * w.bits // 8:e1 * w.bits // 8], q.scales[e0 // w.block:e1 // w.block],
                           q.zps[e0 // w.block:e1 // w.block], e1 - e0, w.bits, w.block)

        def e2e_pipelined():
            start = torch.cuda.Event()
            start.record(stream)
            for st in (s_in, s_cmp, s_out):
                st.wait_event(start)
            for e0, e1 in bounds:
                with torch.cuda.stream(s_in):
                    for r in range(w.P):
                        xs[r][e0:e1].copy_(xs_pinned[r][e0:e1], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
                s_cmp.wait_event(ev_in)
                if variant == "fused":
                    fc.fc_quantized_allreduce([x[e0:e1] for x in xs], w.bits, w.block, y=y[e0:e1],
                                              step1=[qslice(q, e0, e1) for q in s1], step2=qslice(s2, e0, e1),
                                              stream=s_cmp)
                else:
                    fc.fc_quantized_allreduce([x[e0:e1] for x in xs], w.bits, w.block, y=y[e0:e1], stream=s_cmp)
                ev_cmp = torch.cuda.Event()
                ev_cmp.record(s_cmp)
                s_out.wait_event(ev_cmp)
                with torch.cuda.stream(s_out):
                    y_host[e0:e1].copy_(y[e0:e1], non_blocking=True)
            end = torch.cuda.Event()
            end.record(s_out)
            stream.wait_event(end)

        def time_e2e(fn):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(args.e2e_steps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(a.elapsed_time(b) / args.e2e_steps, world)

        ms_copies = time_e2e(e2e_copies)
        y_dev = y.view(torch.int16).cpu()          # the device-buffer call's output
        ms_zero = time_e2e(e2e_zero_copy)
        e2e_exact = bool(torch.equal(y_host.view(torch.int16), y_dev))
        ms_pipe, pipe_exact = None, None
        if bounds:
            y_host.zero_()
            ms_pipe = time_e2e(e2e_pipelined)
            pipe_exact = bool(torch.equal(y_host.view(torch.int16), y_dev))
        # the headline e2e figure is the fastest of the ways a user can call the library on host buffers
        forms = {"zero-copy: the call on page-locked host buffers": ms_zero,
                 "explicit copies: H2D of the inputs, the call on device buffers, D2H of the result": ms_copies}
        if ms_pipe is not None:
            forms[f"pipelined: {len(bounds)} token-row chunks, H2D / fused call / D2H overlapped on three "
                  f"streams"] = ms_pipe
        e2e_mode = min(forms, key=forms.get)
        ms_e2e = forms[e2e_mode]

        in_bytes = w.P * w.n * 2
        value = job_throughput(in_bytes, world, ms)
        value_e2e = job_throughput(in_bytes, world, ms_e2e)
        alg = algorithmic_bytes(w, variant)
        peak, peak_kind = read_peak()
        achieved = alg / (ms * 1e-3) / 1e9
        traffic = read_traffic(w.name, variant)

        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "ms_per_step_median": round(ms_median, 5), "ms_per_step_min": round(ms_min, 5),
            "us_per_allreduce": round(ms * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "description": w.describe(), "variant": variant,
                       "parallelism": f"replicas x{world} (P={w.P} ranks emulated per GPU)",
                       "launch": ("CUDA graph of the timed steps"
                                  if graph is not None or (variant == "staged" and not small and not args.no_graph)
                                  else "stream launches"),
                       "clock_ramp": (f"{ramp_steps} untimed steps (>= {args.ramp_ms:g} ms) enqueued directly before "
                                      f"the timed region, after the {args.warmup} warm-up steps"),
                       "l2": (f"L2 flushed (512 MB write) before each step, each step timed alone"
                              if small else
                              f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB read per step), no flush")},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_kind": f"{peak_kind} copy bandwidth",
                         "algorithmic_bytes_per_launch": alg if variant.startswith("fused") else None,
                         "algorithmic_bytes_per_step": alg},
            "e2e": {"value": round(value_e2e, 3), "unit": "GB/s", "h2d_bytes_per_step": in_bytes,
                    "mode": e2e_mode,
                    "zero_copy_value": round(job_throughput(in_bytes, world, ms_zero), 3),
                    "explicit_copies_value": round(job_throughput(in_bytes, world, ms_copies), 3),
                    "pipelined_value": (round(job_throughput(in_bytes, world, ms_pipe), 3)
                                        if ms_pipe is not None else None),
                    "zero_copy_output_equals_device_path": e2e_exact,
                    "pipelined_output_equals_device_path": pipe_exact,
                    "d2h_bytes_per_step": w.n * 2},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(),
        }

        if staged_extra is not None:
            st_stage_ms, st_step_ms = staged_extra
            st_ms = max_over_ranks(sum(st_stage_ms), world)
            st_alg = algorithmic_bytes(w, "staged")
            st_ach = st_alg / (st_ms * 1e-3) / 1e9
            line["roofline"]["staged"] = {
                "what": f"the staged pipeline (P k_quantize, k_rs, k_ag launches) on the same inputs, {args.steps} "
                        f"steps timed after the fused ones"
                        + ("" if small else ", one replay of a CUDA graph of them after >= --ramp-ms of replays"),
                "algorithmic_bytes_per_step": st_alg, "us_per_allreduce": round(st_ms * 1e3, 2),
                "us_median": round(max_over_ranks(statistics.median(st_step_ms), world) * 1e3, 2),
                "us_min": round(max_over_ranks(min(st_step_ms), world) * 1e3, 2),
                "achieved": round(st_ach, 2), "frac": round(st_ach / peak, 4),
                "kernels_us": {"k_quantize (x P)": round(st_stage_ms[0] * 1e3, 2),
                               "k_rs": round(st_stage_ms[1] * 1e3, 2), "k_ag": round(st_stage_ms[2] * 1e3, 2)},
                "gpu_launches": (w.P + 2) * args.steps}

        if variant == "staged":
            w2b = payload_bytes(w)
            per = {"k_quantize (x P)": (stage_ms[0], w.P * (w.n * 2 + w2b)),
                   "k_rs": (stage_ms[1], w.P * w2b + w2b),
                   "k_ag": (stage_ms[2], w2b + w.n * 2)}
            line["kernels"] = {k: {"us": round(t * 1e3, 2), "algorithmic_bytes": b,
                                   "achieved_gbs": round(b / (t * 1e-3) / 1e9, 1),
                                   "frac": round(b / (t * 1e-3) / 1e9 / peak, 4)}
                               for k, (t, b) in per.items()}

        # ---- N > 1: the method's all-reduce across the job's GPUs (all ranks) ----
        if world > 1 and vi == 0 and not args.no_collective:
            coll = collective_in_line(args, world, rank, local)
            if rank == 0:
                line["collective"] = coll

        # ---- result quality and the CPU baseline (rank 0, N = 1 only) -----------
        if rank == 0:
            torch.cuda.synchronize()
            y_np = y.view(torch.int16).cpu().numpy().view(np.uint16)
            import torch as _t
            wide = [_t.from_numpy(x.view(np.int16)).view(tdt).to(_t.float32).numpy() for x in xs_host]
            S = wide[0].copy()
            for v in wide[1:]:
                S += v                                      # fp32, rank order 0..P-1
            yf = _t.from_numpy(y_np.view(np.int16)).view(tdt).to(_t.float32).numpy().astype(np.float64)
            err = yf - S.astype(np.float64)
            mse = float(np.mean(err * err))
            line["quality"] = {"mse_vs_fp32_sum": mse,
                               "rel_mse": mse / float(np.mean(S.astype(np.float64) ** 2))}
            if world == 1 and not args.no_cpu_baseline and vi == 0:
                import oracle
                rows = args.cpu_rows or w.T
                sub = [x[: rows * w.H] for x in xs_host]
                t0 = time.perf_counter()
                y_ref, _, _ = oracle.allreduce(sub, w.dtype, w.bits, w.block)
                dt = time.perf_counter() - t0
                one = sum(x.size for x in sub) * 2 / dt / 1e9
                line["cpu_baseline"] = {
                    "value": round(one, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                    "sample": f"{rows} of {w.T} token rows per rank, {dt:.1f} s, single thread",
                    "cpu": cpu_model()}
                exact = bool(np.array_equal(y_np[: rows * w.H], y_ref))
                try:   # the same oracle on every host core
                    times, y_team, procs = oracle_team(w, np.stack(sub), rows, 3, host_cores())
                    if procs > 1:
                        dt_team = min(times[1:])
                        line["cpu_baseline"] = {
                            "value": round(sum(x.size for x in sub) * 2 / dt_team / 1e9, 5), "unit": "GB/s",
                            "cores": procs, "kind": "oracle", "cpu": cpu_model(),
                            "sample": (f"{rows} of {w.T} token rows per rank split over {procs} processes "
                                       f"(one per host core), best of 2 runs after 1 warm-up, "
                                       f"{dt_team * 1e3:.1f} ms per run"),
                            "single_thread": line["cpu_baseline"]}
                        exact = exact and bool(np.array_equal(y_np[: y_team.size], y_team))
                except Exception as ex:   # keep the single-thread figure
                    line["cpu_baseline"]["all_cores_error"] = f"{type(ex).__name__}: {ex}"[:200]
                line["quality"]["bit_exact_vs_oracle"] = exact
            print(json.dumps(line), flush=True)

    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
