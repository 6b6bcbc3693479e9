"""The C ABI used from C alone: a gcc-built program (tests/cuda/abi_c_check.c)
allocates device memory with the CUDA driver API, calls the fused all-reduce
and the three staged steps through include/fc.h, and compares every output
and payload byte with the CPU oracle's C definition; it also checks that bad
arguments are refused before launch.  No Python binding or torch memory is
involved in the calls."""
import os
import subprocess

import pytest

import oracle

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PKG = os.path.join(ROOT, "bit_quantized_all_block_b200")
CUDA = "/usr/local/cuda"


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    oracle.build()
    out = str(tmp_path_factory.mktemp("abi") / "abi_c_check")
    odir = os.path.dirname(oracle._LIB)
    subprocess.run(["gcc", "-O1", "-std=c11", "-o", out, os.path.join(HERE, "cuda", "abi_c_check.c"),
                    "-I", os.path.join(CUDA, "include"),
                    "-L", PKG, "-lfc", "-L", odir, "-l:" + os.path.basename(oracle._LIB),
                    "-L", os.path.join(CUDA, "lib64", "stubs"), "-lcuda",
                    f"-Wl,-rpath,{PKG}:{odir}"], check=True)
    return out


@pytest.mark.parametrize("P,dtype,bits,block,n", [
    (4, 0, 8, 128, 4 * 128 * 300 + 4 * 128 * 7),      # several tiles and a ragged tail
    (8, 1, 4, 1024, 8 * 1024 * 19),                    # blocks that span warps
    (2, 0, 4, 32, 2 * 32 * 1001),
    (3, 1, 8, 256, 3 * 256 * 77),
    (4, 0, 8, 128, 4 * 128 * 2),                       # decode-sized message
])
def test_c_caller_matches_the_oracle(program, P, dtype, bits, block, n):
    r = subprocess.run([program, str(P), str(dtype), str(bits), str(block), str(n), str(1000 + P)],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok"), r.stdout
