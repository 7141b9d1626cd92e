"""Attention error margin of the decode under stress, against the oracle.

Short contexts (1 to 3 kf positions), whole-token jumps (probability 0.1, so
most keyframe groups hold a large delta), queries aligned with one cached key
(a dominant score) next to plain N(0, 1) queries, softmax scales from 1/sqrt(128)
up to 1, bf16 and fp32 queries, many seeds.  Every output row must stay within
the row-relative 2e-3 of the oracle's binary64 attention over its own
reconstruction; the worst row of each case is printed.

Source: page "KV 캐시 벡터 양자화와 주의 보존 변환", section "KV 캐시가 왜
병목인가" (the decode step: q.k, softmax, A.V over every cached token).
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from _parity import ATTN_TOL, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
LENS = {32: [1, 2, 3, 5, 8, 13, 21, 31, 32, 33, 47, 63, 64, 65, 80, 96],
        512: [1, 2, 31, 33, 100, 511, 512, 513, 700, 1000, 1023, 1024, 1025, 1200, 1400, 1536]}
SCALES = [1.0 / math.sqrt(128), 0.25, 0.5, 1.0]
WORST = {}


def _queries(K, lens, G, seed, dtype):
    """Half the heads N(0, 1); the other half aligned with one cached key of
    their kv head (scaled to norm sqrt(128) * a, a in {1, 3})."""
    B, Hkv, _, D = K.shape
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hkv * G, D), generator=g, dtype=torch.float64)
    for b in range(B):
        for h in range(Hkv):
            for j in range(G // 2, G):
                p = int(torch.randint(0, lens[b], (1,), generator=g))
                k = K[b, h, p].double()
                a = 1.0 if j % 2 else 3.0
                q[b, h * G + j] = k / k.norm().clamp_min(1e-6) * math.sqrt(D) * a
    return q.to(dtype)


@pytest.mark.parametrize("kf", [32, 512])
@pytest.mark.parametrize("seed", range(6))
def test_attention_stress(orc, dkv_gpu, kf, seed):
    lens = LENS[kf]
    B, Hkv, G = len(lens), 2, 8
    T = max(lens)
    w = S.WORKLOADS["llama3_70b_layer"].with_(B=B, Hkv=Hkv, Hq=Hkv * G, T=T, kf=kf,
                                              jump_p=0.1, seed=4000 + 17 * kf + seed)
    K, V = S.gen_kv(w)
    cache = dkv_gpu.Cache(B, Hkv, T, "delta", kf=kf)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32,
                                                             device=DEV))
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    # the oracle's reconstruction of every sequence, once
    rec = {}
    for b in range(B):
        for h in range(Hkv):
            rec[b, h] = (orc.encode_cache("delta", K[b, h, :lens[b]].float().numpy(), kf)["xhat"],
                         orc.encode_cache("delta", V[b, h, :lens[b]].float().numpy(), kf)["xhat"])
    worst = 0.0
    for qdt in (torch.bfloat16, torch.float32):
        q = _queries(K, lens, G, 77 * seed + kf, qdt)
        qd = q.double().numpy()
        for scale in SCALES:
            out = cache.decode_attn(q.to(DEV), scale)
            torch.cuda.synchronize()
            got = out.cpu().double().numpy()
            ref = np.zeros_like(got)
            for b in range(B):
                for h in range(Hkv):
                    ref[b, h * G:(h + 1) * G] = orc.attn(qd[b, h * G:(h + 1) * G], *rec[b, h],
                                                         scale)
            err = row_rel_err(got, ref)
            e = float(err.max())
            bi, hi = np.unravel_index(int(err.argmax()), err.shape)
            print(f"[stress] kf={kf} seed={seed} q={str(qdt)[6:]} scale={scale:.3f} "
                  f"worst={e:.3e} (b={bi} len={lens[bi]} head={hi})")
            worst = max(worst, e)
            assert e <= ATTN_TOL, (qdt, scale, e, bi, hi)
    WORST[kf, seed] = worst


@pytest.mark.parametrize("kf", [32, 512])
def test_attention_large_magnitudes(orc, dkv_gpu, kf):
    """Keys and values near the top of the fp16 range with whole-token jumps:
    block scales of several thousand.  A weight summed over a keyframe group
    times such a scale would pass the fp16 range if the weights were not
    scaled down; the output must stay finite and within tolerance."""
    lens = LENS[kf]
    B, Hkv, G = len(lens), 2, 8
    T = max(lens)
    w = S.WORKLOADS["llama3_70b_layer"].with_(B=B, Hkv=Hkv, Hq=Hkv * G, T=T, kf=kf,
                                              jump_p=0.2, seed=5100 + kf)
    K, V = S.gen_kv(w)
    K = (K.float() * 600.0).clamp(-6.0e4, 6.0e4).to(torch.float16)
    V = (V.float() * 2000.0).clamp(-6.0e4, 6.0e4).to(torch.float16)
    cache = dkv_gpu.Cache(B, Hkv, T, "delta", kf=kf)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32,
                                                             device=DEV))
    q = S.gen_q(w)
    for scale in (1e-4, 1e-3):
        out = cache.decode_attn(q.to(DEV), scale)
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        got = out.cpu().double().numpy()
        assert np.isfinite(got).all()
        ref = orc.decode_attention("delta", q.double().numpy(), K.float().numpy(),
                                   V.float().numpy(), kf=kf, scale=scale, lengths=lens)
        e = float(row_rel_err(got, ref).max())
        print(f"[stress-large] kf={kf} scale={scale} worst={e:.3e}")
        assert e <= ATTN_TOL, (scale, e)
