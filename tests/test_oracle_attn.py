"""Pins for the oracle's decode-step attention (page 'KV 캐시 벡터 양자화와
주의 보존 변환', section 'KV 캐시가 왜 병목인가': QK^T, softmax, A.V) against
closed forms, invariants and torch's float64 softmax/matmul."""
import math

import numpy as np
import pytest
import torch

import synthetic as S


def _rand(rng, *shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def test_single_token_returns_its_value(orc):
    rng = np.random.default_rng(0)
    q = rng.standard_normal((4, 128))
    k, v = _rand(rng, 1, 128), _rand(rng, 1, 128)
    o = orc.attn(q, k, v, 1 / math.sqrt(128))
    assert np.array_equal(o, np.tile(v.astype(np.float64), (4, 1)))


def test_zero_query_averages_values(orc):
    rng = np.random.default_rng(1)
    k, v = _rand(rng, 37, 128, scale=3), _rand(rng, 37, 128)
    o = orc.attn(np.zeros((2, 128)), k, v, 0.1)
    assert np.allclose(o, v.astype(np.float64).mean(0), rtol=0, atol=1e-14)


def test_two_token_closed_form(orc):
    # s1 - s0 = ln 3 -> weights 1/4, 3/4
    D = 128
    q = np.zeros((1, D)); q[0, 0] = 1.0
    k = np.zeros((2, D), np.float32); k[1, 0] = math.log(3.0) * math.sqrt(D)
    rng = np.random.default_rng(2)
    v = _rand(rng, 2, D)
    o = orc.attn(q, k, v, 1 / math.sqrt(D))
    ref = 0.25 * v[0].astype(np.float64) + 0.75 * v[1].astype(np.float64)
    assert np.allclose(o[0], ref, rtol=0, atol=1e-6)


def test_dominant_score_selects_its_value(orc):
    rng = np.random.default_rng(3)
    D = 128
    k = _rand(rng, 50, D, scale=0.01)
    q = np.ones((1, D))
    k[17] = 3.0                               # score 17 ~ 34 above the rest
    v = _rand(rng, 50, D)
    o = orc.attn(q, k, v, 1 / math.sqrt(D))
    assert np.allclose(o[0], v[17], rtol=0, atol=1e-12)


def test_matches_torch_float64(orc):
    rng = np.random.default_rng(4)
    for T, G in ((1, 1), (5, 3), (300, 8)):
        q = rng.standard_normal((G, 128))
        k, v = _rand(rng, T, 128, scale=2), _rand(rng, T, 128)
        o = orc.attn(q, k, v, 1 / math.sqrt(128))
        s = torch.from_numpy(q) @ torch.from_numpy(k.astype(np.float64)).T / math.sqrt(128)
        ref = torch.softmax(s, dim=-1) @ torch.from_numpy(v.astype(np.float64))
        assert np.allclose(o, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_permutation_and_shift_invariance(orc):
    rng = np.random.default_rng(5)
    q = rng.standard_normal((2, 128))
    k, v = _rand(rng, 64, 128), _rand(rng, 64, 128)
    o = orc.attn(q, k, v, 0.2)
    perm = rng.permutation(64)
    assert np.allclose(orc.attn(q, k[perm], v[perm], 0.2), o, rtol=1e-12, atol=1e-13)
    # a common offset on every key adds the same constant to every score
    # (keys on a 2^-12 grid so that k + 0.5 is exact in binary32)
    k = (np.round(k * 4096) / 4096).astype(np.float32)
    o = orc.attn(q, k, v, 0.2)
    u = np.float32(0.5)
    assert np.allclose(orc.attn(q, k + u, v, 0.2), o, rtol=1e-9, atol=1e-10)


def test_empty_context_gives_zero(orc):
    o = orc.attn(np.ones((1, 128)), np.zeros((0, 128), np.float32),
                 np.zeros((0, 128), np.float32), 1.0)
    assert (o == 0).all()


def test_kf1_delta_attention_equals_fp16_cache(orc):
    w = S.WORKLOADS["llama3_8b_layer"].with_(Hkv=2, Hq=4, T=200)
    K, V = S.gen_kv(w)
    q = S.gen_q(w).double().numpy()
    Kf, Vf = K.float().numpy(), V.float().numpy()
    a = orc.decode_attention("delta", q, Kf, Vf, kf=1, scale=1 / math.sqrt(128))
    b = orc.decode_attention("fp16", q, Kf, Vf, kf=1, scale=1 / math.sqrt(128))
    assert np.array_equal(a, b)


@pytest.mark.parametrize("fmt", ["delta", "q4", "fp16"])
def test_ragged_lengths_use_only_the_prefix(orc, fmt):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, Hkv=1, Hq=2, T=96)
    K, V = S.gen_kv(w)
    q = S.gen_q(w).double().numpy()
    Kf, Vf = K.float().numpy(), V.float().numpy()
    o = orc.decode_attention(fmt, q, Kf, Vf, kf=32, scale=0.1, lengths=[40, 96])
    o40 = orc.decode_attention(fmt, q[:1], Kf[:1, :, :40], Vf[:1, :, :40], kf=32, scale=0.1)
    assert np.array_equal(o[:1], o40)
