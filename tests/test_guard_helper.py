"""The guard-region helper of the GPU bounds tests detects a single byte
written just outside either end of a buffer (checked here on host memory)."""
import pytest

from tests.test_gpu_bounds import G, Guarded


@pytest.mark.parametrize("off", [0, 16])
def test_guard_detects_a_neighbouring_write(off):
    g = Guarded(100, off, device="cpu")
    g.view.fill_(0)                      # writing the buffer itself is fine
    assert g.intact()
    g.raw[g.lo - 1] = 0                  # one byte before
    assert not g.intact()
    g = Guarded(100, off, device="cpu")
    g.raw[g.lo + g.n] = 0                # one byte after
    assert not g.intact()
    g = Guarded(100, off, device="cpu")
    g.raw[G + off + 100 + G - 1] = 1     # the far end of the trailing guard
    assert not g.intact()
