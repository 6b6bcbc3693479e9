"""Failure detection without a fault: the tcgen05 GEMM's bounded mbarrier wait,
given a barrier nothing arrives on, gives up after its time limit (2 s),
raises the CTA's abort flag and returns -- the kernel ends, the context stays
usable (a second kernel runs), and no device trap or hang is involved."""
import ctypes
import os
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_bounded_wait_gives_up(tmp_path):
    from bit_quantized_all_block_b200 import build as B
    so = str(tmp_path / "libwaitcheck.so")
    subprocess.run([B.nvcc(), *B.NVCC_FLAGS, "-shared", "-o", so, os.path.join(HERE, "cuda", "wait_check.cu")],
                   check=True)
    lib = ctypes.CDLL(so)
    out = (ctypes.c_ulonglong * 4)()
    assert lib.fc_check_wait_timeout(out) == 0          # both kernels completed without error
    ok, abort, elapsed_ns, alive = list(out)
    assert ok == 0, "the wait reported success on a barrier nothing arrives on"
    assert abort == 1, "the abort flag was not raised"
    assert 1.9e9 <= elapsed_ns <= 10e9, f"gave up after {elapsed_ns / 1e9:.2f} s"
    assert alive == 42, "the context is not usable after the timeout"
