"""Pins for the oracle's Q4_0 block quantiser and Delta-KV encoder.

Every check here fixes the oracle against something other than itself:
hand-worked examples (tests/golden), closed forms of the block rule, a
brute-force nearest-grid search, numpy's float16 rounding, and invariants the
keyframe + closed-loop delta scheme implies (kf=1 is the F16 cache, a constant
sequence has all-zero deltas, the closed-loop error does not grow with the
distance from the keyframe).  Sources: page 'Delta-KV' (jeff.news article
892), sections 핵심 아이디어, 벤치마크, 컨텍스트 길이에 따른 안정성.
"""
import json
from pathlib import Path

import numpy as np
import pytest
import torch

import synthetic as S

GOLD = json.loads((Path(__file__).parent / "golden" / "quant_worked_examples.json").read_text())


def _block(case):
    v = np.full(32, case.get("fill", 0.0), dtype=np.float32)
    for k, x in case["values_nonzero"].items():
        v[int(k)] = x
    return v


@pytest.mark.parametrize("case", GOLD["blocks"], ids=lambda c: c["name"])
def test_golden_blocks(orc, case):
    v = _block(case)
    d16, codes = orc.quant_block(v)
    assert d16 == int(case["d16"], 16)
    for k, c in case["codes"].items():
        assert codes[int(k)] == c, (k, codes[int(k)], c)
    d = np.float32(np.uint16(d16).view(np.float16))
    for k, x in case.get("dequant", {}).items():
        assert np.float32(int(codes[int(k)]) - 8) * d == np.float32(x)


@pytest.mark.parametrize("case", GOLD["delta_sequences"], ids=lambda c: c["name"])
def test_golden_delta_sequences(orc, case):
    T = len(case["channel0"])
    x = np.zeros((T, case["D"]), dtype=np.float32)
    x[:, 0] = case["channel0"]
    x[:, 1] = case["channel1"]
    s = orc.delta_encode(x, case["kf"])
    for p, h in case["scales"].items():
        assert s.scales[int(p), 0] == int(h, 16), (p, hex(s.scales[int(p), 0]))
    for ch in (0, 1):
        for p, c in case.get(f"codes_ch{ch}", {}).items():
            assert s.codes[int(p), ch] == c
        if f"xhat_ch{ch}" in case:
            assert np.array_equal(s.xhat[:, ch], np.array(case[f"xhat_ch{ch}"], np.float32))
    if "keyframes_ch0" in case:
        assert [int(h, 16) for h in case["keyframes_ch0"]] == [int(v) for v in s.kfr[:, 0]]
    # channels that never move always code 8 on delta rows
    dpos = [p for p in range(T) if p % case["kf"]]
    assert (s.codes[dpos, 2:] == 8).all()


def test_scale_is_fp16_of_m_over_minus_8(orc):
    rng = np.random.default_rng(1)
    for _ in range(300):
        v = (rng.standard_normal(32) * 10.0 ** rng.uniform(-6, 3)).astype(np.float32)
        d16, _ = orc.quant_block(v)
        m = v[np.argmax(np.abs(v))]            # numpy argmax: first index on ties
        ref = (np.float32(m) / np.float32(-8.0)).astype(np.float16).view(np.uint16)
        assert d16 == ref


def test_closed_forms(orc):
    rng = np.random.default_rng(2)
    for _ in range(200):
        i = int(rng.integers(28))       # helpers sit at i+1..i+3, after m
        mag = np.float32(2.0) ** int(rng.integers(-6, 6))
        v = (rng.uniform(-0.9, 0.9, 32) * mag).astype(np.float32)
        v[i] = mag * rng.choice([-1, 1])                 # the unique max: exact d
        v[i + 1] = 0.0
        d16, codes = orc.quant_block(v)
        d = np.float32(np.uint16(d16).view(np.float16))
        assert d == v[i] / np.float32(-8)                # exact scale
        assert codes[i] == 0                            # x = m -> code 0
        assert np.float32(-8) * d == v[i]               # ... dequantises to m
        assert codes[i + 1] == 8                 # x = 0 -> code 8
        # x = -m -> code 15, error |d| (the grid is asymmetric: [-8d, 7d])
        w = v.copy()
        w[i + 2] = -v[i]
        _, c2 = orc.quant_block(w)
        assert c2[i + 2] == 15
        # exact half-way points round up: x = (k + 0.5) d -> code k + 9
        for k in range(-8, 7):
            w = v.copy()
            w[i + 3] = np.float32(k + 0.5) * d
            _, c3 = orc.quant_block(w)
            assert c3[i + 3] == k + 9


def test_codes_are_nearest_grid_point(orc):
    """Brute force: every code is the nearest of the 16 grid values (c-8)d,
    ties towards the larger code, for random blocks over many magnitudes."""
    rng = np.random.default_rng(3)
    for _ in range(2000):
        v = (rng.standard_normal(32) * 10.0 ** rng.uniform(-7, 4)).astype(np.float32)
        d16, codes = orc.quant_block(v)
        d = float(np.uint16(d16).view(np.float16))
        if d == 0.0:
            assert (codes == 8).all()
            continue
        grid = (np.arange(16) - 8) * d
        err = np.abs(v.astype(np.float64)[:, None] - grid[None, :])
        best = err.min(axis=1)
        mine = err[np.arange(32), codes.astype(int)]
        assert (mine <= best + 1e-6 * abs(d)).all()
        # where the choice is not a near-tie it must be the unique best; ties go up
        ratio = v.astype(np.float64) / d
        frac = ratio + 0.5 - np.floor(ratio + 0.5)
        clear = (np.minimum(frac, 1 - frac) > 1e-5)
        up = np.clip(np.floor(ratio + 0.5) + 8, 0, 15)
        assert (codes[clear] == up[clear]).all()


def test_kf1_is_the_fp16_cache(orc):
    w = S.WORKLOADS["tiny"].with_(T=300)
    K, _ = S.gen_kv(w)
    x = K[0, 0].numpy()
    s = orc.delta_encode(x, kf=1)
    ref = x.astype(np.float16).astype(np.float32)
    assert np.array_equal(s.xhat, ref)
    assert (s.codes == 0).all() and (s.scales == 0).all()    # no delta rows at all
    bits, xh16 = orc.f16_encode(x)
    assert np.array_equal(xh16, ref)


def test_constant_sequence_has_zero_deltas(orc):
    rng = np.random.default_rng(4)
    c = rng.standard_normal(128).astype(np.float16).astype(np.float32)
    x = np.tile(c, (100, 1))
    for kf in (2, 7, 32, 512):
        s = orc.delta_encode(x, kf)
        drows = [p for p in range(100) if p % kf]
        assert (s.codes[drows] == 8).all()
        assert np.isin(s.scales[drows], [0x0000, 0x8000]).all()
        assert np.array_equal(s.xhat, x)


def _ulp32(a):
    a = np.abs(a).astype(np.float32)
    return np.spacing(np.maximum(a, np.float32(1e-30))).astype(np.float64)


@pytest.mark.parametrize("kf", [2, 32, 512])
def test_closed_loop_error_bound(orc, kf):
    """|x - xhat| <= |d16|/2 (or about |d16| on the clamped code 15) plus fp32
    rounding, whatever the distance from the keyframe."""
    w = S.WORKLOADS["llama3_8b_layer"].with_(Hkv=2, T=1024, kv_dtype=torch.float32)
    K, V = S.gen_kv(w)
    for x in (K[0, 0].numpy(), V[0, 1].numpy()):
        s = orc.delta_encode(x, kf)
        T, D = x.shape
        pos = np.array([p for p in range(T) if p % kf])
        d = np.abs(s.scales[pos].view(np.float16).astype(np.float64))      # [n, 4]
        dch = np.repeat(d, 32, axis=1)                                     # per channel
        code = s.codes[pos].astype(int)
        # clamped code 15: |x/d16| may exceed 8 by the fp16 rounding of d
        # (relative 2^-11), so the bound there is |d16| (1 + 8 * 2^-11)
        lim = np.where(code == 15, 1.0 + 8 * 2.0 ** -11, 0.5) * dch * (1 + 1e-6)
        err = np.abs(x[pos].astype(np.float64) - s.xhat[pos].astype(np.float64))
        tol = lim + 4 * np.maximum(_ulp32(x[pos]), _ulp32(s.xhat[pos]))
        assert (err <= tol).all(), float((err - tol).max())
        if kf == 512:
            # no drift: relative to the block scale, the error late in a group is
            # no larger than early on (an open-loop encoder grows like sqrt(j))
            j = pos % kf
            rel = err / np.maximum(dch, 1e-30)
            early = rel[(j >= 1) & (j < 128)].mean()
            late = rel[j >= 384].mean()
            assert late < 1.25 * early, (late, early)


@pytest.mark.parametrize("kf", [1, 3, 32, 33, 512])
def test_decode_reproduces_encoder_state(orc, kf):
    w = S.WORKLOADS["llama3_8b_layer"].with_(Hkv=1, T=700)
    K, _ = S.gen_kv(w)
    x = K[0, 0].float().numpy()
    s = orc.delta_encode(x, kf)
    xr = orc.delta_decode(700, kf, s.kfr, s.scales, s.codes)
    assert np.array_equal(xr.view(np.uint32), s.xhat.view(np.uint32))
    assert np.array_equal(s.state, s.xhat[-1])


def test_append_in_pieces_equals_one_encode(orc):
    w = S.WORKLOADS["ragged_long"].with_(B=1, Hkv=1, T=400, ragged=None)
    K, _ = S.gen_kv(w)
    x = K[0, 0].float().numpy()
    whole = orc.delta_encode(x, 32)
    part = orc.DeltaSeq(400, 128, 32)
    cuts = [0, 1, 2, 31, 32, 33, 100, 255, 256, 257, 399, 400]
    for a, b in zip(cuts[:-1], cuts[1:]):
        part.append(x[a:b])
    for f in ("kfr", "scales", "codes", "xhat", "state"):
        assert np.array_equal(getattr(part, f), getattr(whole, f)), f


def test_mse_delta_vs_q4_vs_fp16(orc):
    """The pages argue deltas span ~100x less range, hence ~10^4x less
    quantisation error than Q4_0 on absolute values; on a pure 1%-step random
    walk the MSE ratio lands in that neighbourhood (a loose sanity band)."""
    w = S.WORKLOADS["tiny"].with_(T=2048, kv_dtype=torch.float16)
    K, _ = S.gen_kv(w)
    x = K[0, 0].float().numpy()
    e_delta = ((orc.encode_cache("delta", x, 32)["xhat"] - x) ** 2).mean()
    e_q4 = ((orc.encode_cache("q4", x)["xhat"] - x) ** 2).mean()
    e_f16 = ((orc.encode_cache("fp16", x)["xhat"] - x) ** 2).mean()
    assert e_f16 == 0.0            # the inputs are fp16 already
    assert 1e3 < e_q4 / e_delta < 1e5, e_q4 / e_delta
