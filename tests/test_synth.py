"""Seeded input generator: determinism, prefix sampling, recipe shape."""
import numpy as np

from bit_quantized_all_block_b200 import synth


def test_deterministic_and_prefix():
    a = synth.partials(3, 16, 512, synth.FP16, 0.01, 20.0, seed=0)
    b = synth.partials(3, 16, 512, synth.FP16, 0.01, 20.0, seed=0)
    assert np.array_equal(a, b)
    head = synth.partials(3, 16, 512, synth.FP16, 0.01, 20.0, seed=0, rows=5)
    assert np.array_equal(head, a[:, :5 * 512])
    c = synth.partials(3, 16, 512, synth.FP16, 0.01, 20.0, seed=1)
    assert not np.array_equal(a, c)


def test_outlier_channels_and_divisibility():
    x = synth.partials(2, 256, 1024, synth.FP16, 0.01, 20.0).view(np.float16).astype(np.float32)
    ch = np.abs(x.reshape(2, 256, 1024)).mean(axis=(0, 1))
    # ~10 channels carry a 20x scale: the top-10 channel means dominate the median
    top = np.sort(ch)[-10:]
    assert top.min() > 8 * np.median(ch)
    for w in (synth.SMALL_P2, synth.PREFILL_70B_INT8, synth.PREFILL_70B_INT4, synth.DECODE_P4,
              *synth.BLOCK_SWEEP_8B, *synth.message_sweep(8)):
        assert w.n % (w.P * w.block) == 0, w.name


def test_message_sweep_sizes():
    sw = synth.message_sweep(4)
    assert [w.n * 2 for w in sw][0] == 16 * 1024 and sw[-1].n * 2 == 1 << 30 and len(sw) == 17
