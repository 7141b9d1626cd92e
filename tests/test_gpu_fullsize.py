"""Parity at the workloads' full sizes, in the launch configuration bench.py
times: the whole cache is encoded and decoded on the GPU; sampled (batch,
kv-head) sequences are checked against the CPU oracle (codes, scales,
keyframes and closed-loop state bit-exact; attention of the sampled query
heads within the 2e-3 row-relative tolerance)."""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from _parity import ATTN_TOL, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check(orc, dkv, w, lens, n_append=0, samples=((0, 0),)):
    """Encode (and append) w on the GPU, decode once, compare sampled sequences."""
    Tg = max(lens)
    K = torch.empty((w.B, w.Hkv, Tg, w.D), dtype=w.kv_dtype, device=DEV)
    V = torch.empty_like(K)
    for b in range(w.B):
        K[b], V[b] = S.gen_kv_one(w, b, Tg, device=DEV)
    q = S.gen_q(w, device=DEV)
    cache = dkv.Cache(w.B, w.Hkv, Tg, "delta", kf=w.kf)
    enc_lens = torch.tensor([L - n_append for L in lens], dtype=torch.int32, device=DEV)
    cache.encode(K, V, seq_lens=enc_lens)
    for i in range(n_append):
        # token i of the appended block sits at position enc_len + i of each sequence
        idx = (enc_lens.long() + i).clamp(max=Tg - 1)
        kn = torch.stack([K[b, :, idx[b]] for b in range(w.B)])[:, :, None].contiguous()
        vn = torch.stack([V[b, :, idx[b]] for b in range(w.B)])[:, :, None].contiguous()
        cache.append(kn, vn)
    scale = 1.0 / math.sqrt(w.D)
    out = cache.decode_attn(q, scale)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == list(lens)
    ex = cache.export()
    G = w.Hq // w.Hkv
    for (b, h) in samples:
        L = lens[b]
        for t, X in enumerate((K, V)):
            x = X[b, h, :L].float().cpu().numpy()
            ref = orc.delta_encode(x, w.kf, cap=Tg)
            codes = ex["codes"][b, h, t].cpu().numpy()
            scales = ex["scales"][b, h, t].cpu().numpy().view(np.uint16)
            kfr = ex["keyframes"][b, h, t].cpu().numpy().view(np.uint16)
            assert np.array_equal(codes[:L], ref.codes[:L]), (b, h, t, "codes")
            assert np.array_equal(scales[:L], ref.scales[:L]), (b, h, t, "scales")
            ng = -(-L // w.kf)
            assert np.array_equal(kfr[:ng], ref.kfr[:ng]), (b, h, t, "keyframes")
            st = ex["state"][b, h, t].cpu().numpy()
            assert np.array_equal(st.view(np.uint32), ref.state.view(np.uint32)), (b, h, t, "state")
            if t == 0:
                kh = ref.xhat[:L]
            else:
                vh = ref.xhat[:L]
        qb = q[b, h * G:(h + 1) * G].double().cpu().numpy()
        o_ref = orc.attn(qb, kh, vh, scale)
        err = row_rel_err(out[b, h * G:(h + 1) * G].cpu().numpy(), o_ref).max()
        print(f"[fullsize] {w.name} kf={w.kf} B={w.B} T={lens} sample=({b},{h}) "
              f"max_row_rel_err={err:.3e}")
        assert err <= ATTN_TOL, (b, h, err)


def test_llama3_70b_layer_full(orc, dkv_gpu):
    w = S.WORKLOADS["llama3_70b_layer"]
    _check(orc, dkv_gpu, w, [w.T] * w.B, samples=((0, 0), (7, 3), (15, 7)))


def test_llama3_8b_layer_full(orc, dkv_gpu):
    w = S.WORKLOADS["llama3_8b_layer"]
    _check(orc, dkv_gpu, w, [w.T], samples=tuple((0, h) for h in range(w.Hkv)))


@pytest.mark.parametrize("kf,gen", [(32, "walk"), (512, "walk"), (32, "repeat")])
def test_batched_decode_full(orc, dkv_gpu, kf, gen):
    w = S.WORKLOADS["batched_decode"].with_(kf=kf, gen=gen)
    _check(orc, dkv_gpu, w, [w.T] * w.B, samples=((0, 0), (11, 5)))


@pytest.mark.parametrize("kf", [32, 128, 512])
def test_ragged_long_with_appends(orc, dkv_gpu, kf):
    w = S.WORKLOADS["ragged_long"].with_(kf=kf)
    lens = [L + w.n_append for L in S.gen_lengths(w)]
    _check(orc, dkv_gpu, w, lens, n_append=w.n_append, samples=((0, 0), (3, 6)))


def test_large_block_append_mid_group(orc, dkv_gpu):
    """One append of 4000 tokens per sequence onto a prefix that ends inside a
    keyframe group, at the batched-decode shape: enough closed loops that the
    append runs one lane per loop (the prefill kernel), continuing from the
    stored reconstruction."""
    w = S.WORKLOADS["batched_decode"].with_(T=16384 - 37)
    Tg = w.T
    n = 4000
    K = torch.empty((w.B, w.Hkv, Tg, w.D), dtype=w.kv_dtype, device=DEV)
    V = torch.empty_like(K)
    for b in range(w.B):
        K[b], V[b] = S.gen_kv_one(w, b, Tg, device=DEV)
    cache = dkv_gpu.Cache(w.B, w.Hkv, Tg, "delta", kf=w.kf)
    cache.encode(K[:, :, :Tg - n].contiguous(), V[:, :, :Tg - n].contiguous())
    cache.append(K[:, :, Tg - n:].contiguous(), V[:, :, Tg - n:].contiguous())
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == [Tg] * w.B
    ex = cache.export()
    for (b, h) in ((0, 0), (9, 4), (15, 7)):
        for t, X in enumerate((K, V)):
            ref = orc.delta_encode(X[b, h].float().cpu().numpy(), w.kf, cap=Tg)
            assert np.array_equal(ex["codes"][b, h, t].cpu().numpy(), ref.codes), (b, h, t)
            assert np.array_equal(ex["scales"][b, h, t].cpu().numpy().view(np.uint16), ref.scales)
            ng = -(-Tg // w.kf)
            assert np.array_equal(ex["keyframes"][b, h, t].cpu().numpy().view(np.uint16)[:ng],
                                  ref.kfr[:ng])
            assert np.array_equal(ex["state"][b, h, t].cpu().numpy().view(np.uint32),
                                  ref.state.view(np.uint32))


# ---------------------------------------------------------------------------
# the other decode forms bench.py times at the headline shape, at full size
# ---------------------------------------------------------------------------
def _headline_kv(w, T):
    K = torch.empty((w.B, w.Hkv, T, w.D), dtype=w.kv_dtype, device=DEV)
    V = torch.empty_like(K)
    for b in range(w.B):
        K[b], V[b] = S.gen_kv_one(w, b, T, device=DEV)
    return K, V


def _sample_refs(orc, K, V, ex, b, h, L, kf, cap):
    """The oracle's encoding of sequence (b, h): the stored fields must equal
    it bit for bit; returns its reconstruction of K and V."""
    xh = []
    for t, X in enumerate((K, V)):
        ref = orc.delta_encode(X[b, h, :L].float().cpu().numpy(), kf, cap=cap)
        if ex is not None:
            assert np.array_equal(ex["codes"][b, h, t].cpu().numpy()[:L], ref.codes[:L]), (b, h, t)
            assert np.array_equal(ex["scales"][b, h, t].cpu().numpy().view(np.uint16)[:L],
                                  ref.scales[:L]), (b, h, t)
            ng = -(-L // kf)
            assert np.array_equal(ex["keyframes"][b, h, t].cpu().numpy().view(np.uint16)[:ng],
                                  ref.kfr[:ng]), (b, h, t)
            assert np.array_equal(ex["state"][b, h, t].cpu().numpy().view(np.uint32),
                                  ref.state.view(np.uint32)), (b, h, t)
        xh.append(ref.xhat[:L])
    return xh


def test_llama3_70b_layer_fused_append_full(orc, dkv_gpu):
    """dkv_append_decode_attn as bench.py's fused step: one new token per
    sequence onto 32767 encoded ones, quantised inside the split kernel, then
    attention over all 32768."""
    w = S.WORKLOADS["llama3_70b_layer"]
    T = w.T
    K, V = _headline_kv(w, T)
    cache = dkv_gpu.Cache(w.B, w.Hkv, T, "delta", kf=w.kf)
    cache.encode(K[:, :, :T - 1].contiguous(), V[:, :, :T - 1].contiguous())
    q = S.gen_q(w, device=DEV)
    scale = 1.0 / math.sqrt(w.D)
    out = cache.append_decode_attn(K[:, :, T - 1:].contiguous(), V[:, :, T - 1:].contiguous(), q,
                                   scale)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == [T] * w.B
    ex = cache.export()
    G = w.Hq // w.Hkv
    for (b, h) in ((0, 0), (6, 2), (15, 7)):
        kh, vh = _sample_refs(orc, K, V, ex, b, h, T, w.kf, T)
        o_ref = orc.attn(q[b, h * G:(h + 1) * G].double().cpu().numpy(), kh, vh, scale)
        err = row_rel_err(out[b, h * G:(h + 1) * G].cpu().numpy(), o_ref).max()
        print(f"[fullsize-fused] sample=({b},{h}) max_row_rel_err={err:.3e}")
        assert err <= ATTN_TOL, (b, h, err)


def test_llama3_70b_layer_paged_full(orc, dkv_gpu):
    """The headline decode through a paged cache: pages of 16 keyframe groups
    in a shuffled pool (bench.py's paged comparator)."""
    w = S.WORKLOADS["llama3_70b_layer"]
    T = w.T
    K, V = _headline_kv(w, T)
    cache = dkv_gpu.Cache(w.B, w.Hkv, T, "delta", kf=w.kf, page_groups=16, page_seed=7)
    cache.encode(K, V)
    q = S.gen_q(w, device=DEV)
    scale = 1.0 / math.sqrt(w.D)
    out = cache.decode_attn(q, scale)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    ex = cache.export()
    G = w.Hq // w.Hkv
    for (b, h) in ((1, 1), (14, 6)):
        kh, vh = _sample_refs(orc, K, V, ex, b, h, T, w.kf, T)
        o_ref = orc.attn(q[b, h * G:(h + 1) * G].double().cpu().numpy(), kh, vh, scale)
        err = row_rel_err(out[b, h * G:(h + 1) * G].cpu().numpy(), o_ref).max()
        print(f"[fullsize-paged] sample=({b},{h}) max_row_rel_err={err:.3e}")
        assert err <= ATTN_TOL, (b, h, err)


def test_llama3_70b_layer_two_queries_full(orc, dkv_gpu):
    """dkv_decode_attn_mq with 2 causal queries per sequence at the headline
    shape (bench.py's 2-query comparator: 16 virtual heads per kv head)."""
    w = S.WORKLOADS["llama3_70b_layer"]
    T = w.T
    K, V = _headline_kv(w, T)
    cache = dkv_gpu.Cache(w.B, w.Hkv, T, "delta", kf=w.kf)
    cache.encode(K, V)
    g = torch.Generator().manual_seed(2)
    Q = torch.randn((w.B, 2, w.Hq, w.D), generator=g).to(w.q_dtype)
    scale = 1.0 / math.sqrt(w.D)
    out = cache.decode_attn_mq(Q.to(DEV), scale)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    G = w.Hq // w.Hkv
    for (b, h) in ((3, 4), (12, 0)):
        kh, vh = _sample_refs(orc, K, V, None, b, h, T, w.kf, T)
        for t in range(2):
            L = T - (1 - t)                          # query t sees the positions before L
            o_ref = orc.attn(Q[b, t, h * G:(h + 1) * G].double().numpy(), kh[:L], vh[:L], scale)
            err = row_rel_err(out[b, t, h * G:(h + 1) * G].cpu().numpy(), o_ref).max()
            print(f"[fullsize-mq] sample=({b},{h}) query={t} max_row_rel_err={err:.3e}")
            assert err <= ATTN_TOL, (b, h, t, err)
