"""The tcgen05 GEMM with the fused step-1 quantizer (fc_gemm_quantize).

partial = a @ w.T is a contraction on the tensor cores with fp32 accumulation
in the hardware's order, so it is checked against the exact product (numpy
float64 of the exactly widened 16-bit inputs) within a bound derived from the
arithmetic: one rounding to the 16-bit type (half an ulp, 2^-9 relative for
bf16 / 2^-12 for fp16, doubled for safety) plus fp32 accumulation error
K * 2^-22 * sum|a_k w_k|.  The payload is a discrete function of the partial,
so it must equal the oracle's quantization of the GPU's own partial bit for
bit; and a P-rank pipeline (GEMM+quantize per rank, then reduce-scatter and
all-gather) must equal the oracle's all-reduce of those partials."""
import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from tests.gpu_util import assert_payload_equal, assert_y_equal

pytestmark = pytest.mark.gpu


def operands(M, N, K, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g).to(dtype)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(dtype)
    return a, w


def check_partial(p_gpu, a, w, dtype):
    a64 = a.double().numpy()
    w64 = w.double().numpy()
    ref = a64 @ w64.T
    S = np.abs(a64) @ np.abs(w64).T
    K = a.shape[1]
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -11
    got = p_gpu.double().cpu().numpy()
    bound = rel * np.abs(ref) + K * 2.0 ** -22 * S + 1e-30
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} partial values outside the bound, worst {np.max(np.abs(got - ref) - bound)}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("block", [32, 64, 128, 256])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (256, 512, 192), (1024, 1536, 256)])
def test_gemm_quantize_small(dtype, bits, block, M, N, K):
    a, w = operands(M, N, K, dtype, seed=M + N + K + bits + block)
    ad, wd = a.cuda(), w.cuda()
    partial = torch.empty(M, N, dtype=dtype, device="cuda")
    q, p, status = fc.fc_gemm_quantize(ad, wd, bits, block, partial=partial)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    check_partial(p, a, w, dtype)
    odt = oracle.BF16 if dtype == torch.bfloat16 else oracle.FP16
    p_bits = p.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    ref = oracle.quantize(p_bits, odt, bits, block)
    assert_payload_equal(q, ref, "fused payload")


def test_gemm_persistent_many_tiles():
    """More tiles than SMs: every CTA cycles through both TMEM accumulators."""
    M, N, K = 4096, 4096, 512
    a, w = operands(M, N, K, torch.bfloat16, seed=7)
    ad, wd = a.cuda(), w.cuda()
    q, p, status = fc.fc_gemm_quantize(ad, wd, 8, 128, partial=torch.empty(M, N, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    rows = np.r_[0:8, 1000:1008, M - 8:M]
    check_partial(p[rows].cpu(), a[rows], w, torch.bfloat16)
    ref = oracle.quantize(p.view(torch.int16).cpu().numpy().view(np.uint16).ravel(), oracle.BF16, 8, 128)
    assert_payload_equal(q, ref, "payload")
    # the partial-only mode writes the same partial
    _, p2, st2 = fc.fc_gemm_quantize(ad, wd, 8, 128, quantize=False)
    torch.cuda.synchronize()
    assert int(st2[0].item()) == 0 and torch.equal(p2.view(torch.int16), p.view(torch.int16))


@pytest.mark.parametrize("bits", [8, 4])
def test_tp_pipeline(bits):
    """P ranks: fused GEMM+quantize, then reduce-scatter and all-gather."""
    P, M, N, Kr, block = 4, 512, 1024, 128, 128
    outs, parts = [], []
    for r in range(P):
        a, w = operands(M, N, Kr, torch.bfloat16, seed=100 + r)
        q, p, st = fc.fc_gemm_quantize(a.cuda(), w.cuda(), bits, block,
                                       partial=torch.empty(M, N, dtype=torch.bfloat16, device="cuda"))
        outs.append(q)
        parts.append(p)
    q2 = fc.fc_rs_dequant_sum_requant(outs, bits, block)
    y = fc.fc_ag_dequant(q2, torch.bfloat16)
    torch.cuda.synchronize()
    xs = [p.view(torch.int16).cpu().numpy().view(np.uint16).ravel() for p in parts]
    y_ref, p1_ref, p2_ref = oracle.allreduce(xs, oracle.BF16, bits, block)
    assert_payload_equal(q2, p2_ref, "step-2 payload")
    assert_y_equal(y, y_ref, "all-reduced output")


def test_gemm_validation():
    a = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda")
    for kw in [dict(block=512), dict(block=16), dict(bits=3)]:
        with pytest.raises(fc.FCError):
            fc.fc_gemm_quantize(a, w, kw.get("bits", 8), kw.get("block", 128))
    with pytest.raises(fc.FCError):
        fc.fc_gemm_quantize(a[:, :32].contiguous(), w[:, :32].contiguous(), 8, 128)   # K % 64


def device_operands(M, N, K, dtype, seed):
    """Seeded operands drawn on the device (the large shapes), with host copies."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    a = torch.randn(M, K, device="cuda", generator=g).to(dtype)
    w = (torch.randn(N, K, device="cuda", generator=g) / K ** 0.5).to(dtype)
    return a, w


def sample_rows(M, seed):
    """First and last rows, both sides of 128- and 256-row tile edges, random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, 1, 127, 128, 255, 256, M // 2 - 1, M // 2, M - 129, M - 128, M - 2, M - 1}
    rows |= set(int(r) for r in rng.integers(0, M, size=12))
    return np.array(sorted(r for r in rows if 0 <= r < M))


@pytest.mark.parametrize("M,bits,block,dtype", [
    (8192, 8, 128, torch.bfloat16),    # the benchmarked o_proj shape per rank: SM-pair kernel (M % 256 == 0)
    (8192, 4, 256, torch.bfloat16),    # SM pairs, blocks of a whole tile row
    (8064, 8, 128, torch.bfloat16),    # M % 256 != 0: the one-SM kernel
    (8064, 4, 64, torch.bfloat16),
    (8192, 8, 128, torch.float16),     # fp16 operands on both kernels
    (8064, 4, 256, torch.float16),
], ids=["pair-int8-b128", "pair-int4-b256", "onesm-int8-b128", "onesm-int4-b64", "pair-fp16-int8-b128",
        "onesm-fp16-int4-b256"])
def test_gemm_at_the_benchmarked_shape(M, bits, block, dtype):
    """N = 8192, K = 2048 (70B-shaped o_proj slice of one rank of 4): the whole
    payload equals the oracle's quantization of the GPU's partial; sampled rows
    of the partial lie within the accumulation bound of the exact product."""
    N, K = 8192, 2048
    a, w = device_operands(M, N, K, dtype, seed=M + bits + block)
    partial = torch.empty(M, N, dtype=dtype, device="cuda")
    q, p, status = fc.fc_gemm_quantize(a, w, bits, block, partial=partial)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    rows = sample_rows(M, seed=M)
    check_partial(p[rows].cpu(), a[rows].cpu(), w.cpu(), dtype)
    odt = oracle.BF16 if dtype == torch.bfloat16 else oracle.FP16
    ref = oracle.quantize(p.view(torch.int16).cpu().numpy().view(np.uint16).ravel(), odt, bits, block)
    assert_payload_equal(q, ref, "payload")


def test_gemm_down_projection_depth_sampled_rows():
    """K = 7168 (the down-projection slice): sampled rows of the partial within
    the accumulation bound, and those rows' codes, scales and zero-points equal
    the oracle's quantization of the same rows of the GPU partial."""
    M, N, K, bits, block, dtype = 8192, 8192, 7168, 8, 128, torch.bfloat16
    a, w = device_operands(M, N, K, dtype, seed=71)
    partial = torch.empty(M, N, dtype=dtype, device="cuda")
    q, p, status = fc.fc_gemm_quantize(a, w, bits, block, partial=partial)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    rows = sample_rows(M, seed=7)
    check_partial(p[rows].cpu(), a[rows].cpu(), w.cpu(), dtype)
    nb = N // block
    codes = q.codes.view(M, N).cpu().numpy()
    scales = q.scales.view(M, nb).cpu().numpy()
    zps = q.zps.view(M, nb).cpu().numpy()
    for r in rows:
        ref = oracle.quantize(p[r].view(torch.int16).cpu().numpy().view(np.uint16), oracle.BF16, bits, block)
        assert np.array_equal(codes[r], ref.codes), f"row {r}: codes differ"
        assert np.array_equal(scales[r].view(np.uint32), ref.scales.view(np.uint32)), f"row {r}: scales differ"
        assert np.array_equal(zps[r], ref.zps), f"row {r}: zero-points differ"
