"""Pins for the oracle's long-range reference encoder (the training-free part
of DeltaKV: fp16 references at a fixed stride, every other token the Q4_0
residual against the mean of its most similar earlier references; page
'DeltaKV' summary, sections 2 (long-range inter-token similarity) and A
(Strided Reference Selection, Residual Encoding, Reconstruction), and
'양자화 친화성' in section 4).

Each check fixes the encoder against something other than itself: numpy's
float16 rounding (stride 1 stores every token as fp16), the already pinned
Q4_0 comparator (one reference: the residual against it is plain Q4_0), exact
repeats (a token equal to a stored reference costs nothing), a brute-force
distance ranking in numpy, and the block rule's error bound.
"""
import numpy as np
import pytest


def _rand(T, D, seed):
    return np.random.RandomState(seed).randn(T, D).astype(np.float32)


def test_stride_one_is_the_fp16_cache(orc):
    x = _rand(37, 64, 1)
    o = orc.lr_encode(x, 1, 3)
    assert (o["ref"] == -1).all()
    assert np.array_equal(o["xhat"], x.astype(np.float16).astype(np.float32))
    assert np.array_equal(o["kfr"], x.astype(np.float16).view(np.uint16))
    assert not o["codes"].any() and not o["scales"].any()


@pytest.mark.parametrize("m", [1, 4])
def test_single_reference_is_q4_of_the_residual(orc, m):
    """With the stride past the end only token 0 is a reference: every other
    token's residual is taken against it, so its codes, scales and
    reconstruction are the plain Q4_0 comparator's on x - fp16(x_0)."""
    x = _rand(29, 128, 2)
    o = orc.lr_encode(x, 1000, m)
    k0 = x[0].astype(np.float16).astype(np.float32)
    sc, co, xh = orc.q4_encode(x[1:] - k0[None])
    assert (o["ref"][1:, 0] == 0).all() and (o["ref"][1:, 1:] == -1).all()
    assert np.array_equal(o["scales"][1:], sc)
    assert np.array_equal(o["codes"][1:], co)
    assert np.array_equal(o["xhat"][1:], k0[None] + xh)


def test_exact_repeat_of_a_reference_is_lossless(orc):
    """A token equal to an earlier stored reference (fp16-exact values) picks
    it (distance 0) and has a zero residual: every code 8, every scale zero
    (-0: d = m / -8 of an all-zero block), the reconstruction exact."""
    s, T, D = 8, 64, 64
    x = _rand(T, D, 3).astype(np.float16).astype(np.float32)
    for p, r in ((13, 8), (41, 16), (50, 0), (63, 40)):
        x[p] = x[r]
    o = orc.lr_encode(x, s, 1)
    for p, r in ((13, 8), (41, 16), (50, 0), (63, 40)):
        assert o["ref"][p, 0] == r // s
        assert (o["codes"][p] == 8).all()
        assert (o["scales"][p].view(np.float16) == 0).all()
        assert np.array_equal(o["xhat"][p], x[p])


@pytest.mark.parametrize("s,m", [(4, 1), (4, 3), (7, 2), (16, 5)])
def test_choice_matches_a_brute_force_ranking(orc, s, m):
    """The chosen references are the m earlier stride positions whose stored
    (fp16) values are nearest in squared Euclidean distance, ranked here with
    numpy in binary64; their mean reproduces the reconstruction."""
    T, D = 70, 64
    x = _rand(T, D, 4 + s + m)
    o = orc.lr_encode(x, s, m)
    kv = x[::s].astype(np.float16).astype(np.float64)
    for p in range(T):
        if p % s == 0:
            assert (o["ref"][p] == -1).all()
            continue
        cand = np.arange(0, p, s) // s
        d = ((x[p].astype(np.float64)[None] - kv[cand]) ** 2).sum(axis=1)
        order = sorted(range(len(cand)), key=lambda i: (d[i], cand[i]))
        want = sorted(int(cand[i]) for i in order[:m])
        got = [int(g) for g in o["ref"][p] if g >= 0]
        assert got == want, (p, got, want)
        mean = kv[want].mean(axis=0)
        d16 = o["scales"][p].view(np.float16).astype(np.float64)
        step = (o["codes"][p].astype(np.float64) - 8) * np.repeat(d16, 32)
        assert np.allclose(o["xhat"][p] - step, mean, rtol=0, atol=1e-5)


def test_reconstruction_error_within_the_block_step(orc):
    """Per element |x^ - x| <= |d|/2 for codes inside the grid, <= |d| where
    the code was clamped at 15 (the Q4_0 rule's range ends at +7 d)."""
    x = _rand(90, 128, 9) * 3
    o = orc.lr_encode(x, 16, 2)
    d = np.repeat(o["scales"].view(np.float16).astype(np.float64), 32, axis=1)
    err = np.abs(o["xhat"].astype(np.float64) - x)
    ref_rows = np.arange(90) % 16 == 0
    lim = np.where(o["codes"] == 15, np.abs(d), np.abs(d) / 2) * (1 + 1e-6) + 1e-7
    assert (err[~ref_rows] <= lim[~ref_rows]).all()


def test_attention_over_stride_one_is_the_fp16_cache(orc):
    """A decode step over the long-range format with stride 1 (every token a
    fp16 reference) is the decode step over the fp16 cache."""
    rs = np.random.RandomState(12)
    K = rs.randn(2, 2, 40, 64).astype(np.float32)
    V = rs.randn(2, 2, 40, 64).astype(np.float32)
    q = rs.randn(2, 4, 64)
    a = orc.decode_attention("lr", q, K, V, kf=1, scale=0.125)
    b = orc.decode_attention("fp16", q, K, V, kf=1, scale=0.125)
    assert np.array_equal(a, b)
