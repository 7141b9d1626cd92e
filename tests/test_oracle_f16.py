"""Pins for the oracle's binary16 conversions against numpy's float16 (a
library implementation of IEEE 754 binary16 with round-to-nearest-even)."""
import numpy as np


def test_f16_to_f32_all_bit_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.f16_bits_to_f32(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_rounding(orc):
    rng = np.random.default_rng(7)
    parts = [
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000)).astype(np.float32),
        # exact ties between neighbouring binary16 values (round half to even)
        (np.arange(1, 2048, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -10),
        (np.arange(1, 1024, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -24),
        np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 65536.0, 1e6, -1e6, 6.1e-5,
                  6.103515625e-05, 5.96e-8, 2.98e-8, 2.9802322e-8, 1e-9, -1e-9,
                  np.inf, -np.inf], dtype=np.float32),
    ]
    x = np.concatenate(parts)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    ours = orc.f32_to_f16_bits(x)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), int(ours[i]), int(ref[i])) for i in bad[:5]]
