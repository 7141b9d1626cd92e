"""The corner-case sequences of ``_edge`` really hit every corner of the block
rule (checked on the CPU, from the oracle's encoding of them), so the GPU
tests that feed them to the CUDA writers exercise what they claim to."""
import numpy as np
import pytest

import _edge as E


@pytest.mark.parametrize("kf", [2, 32, 33, 512])
def test_edge_sequences_cover_every_corner(orc, kf):
    T = 1100 if kf == 512 else 300
    tot = {}
    for seed in (1, 2):
        x = E.edge_sequence(orc, T, kf, seed)
        assert np.isfinite(x).all()
        kfr_rows = x[::kf]
        assert np.array_equal(kfr_rows.astype(np.float16).astype(np.float32), kfr_rows)
        c = E.coverage(x, kf, orc.delta_encode(x, kf))
        for k, v in c.items():
            tot[k] = tot.get(k, 0) + v
    for k in ("tie", "tie_high", "zero_block", "half", "clamp15", "clamp0", "sub_d",
              "zero_d_nonzero"):
        assert tot[k] > 0, (k, tot)


def test_designed_deltas_are_realised_exactly(orc):
    """In the dyadic regime the closed-loop delta the oracle quantises is the
    designed block itself: re-deriving it from x and the reconstruction gives
    values on the designed grid (multiples of 2^-9 of magnitude <= 2)."""
    kf = 32
    x = E.edge_sequence(orc, 320, kf, 5)
    enc = orc.delta_encode(x, kf)
    hits = 0
    for p in range(1, 320):
        if p % kf == 0:
            continue
        delta = (x[p] - enc.xhat[p - 1]).astype(np.float32)
        for j in range(4):
            v = delta[32 * j:32 * j + 32].astype(np.float64)
            if np.abs(v).max() <= 2.0 and np.abs(v).max() >= 2.0 ** -3:
                if np.all(v * 512 == np.round(v * 512)):
                    hits += 1
    assert hits > 100


def test_constant_sequence_has_zero_deltas(orc):
    x = E.constant_sequence(100, 3)
    s = orc.delta_encode(x, 32)
    rows = [p for p in range(100) if p % 32]
    assert (s.codes[rows] == 8).all()
    assert (s.scales[rows] == 0x8000).all()
