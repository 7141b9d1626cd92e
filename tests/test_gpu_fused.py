"""GPU parity of the fused append + decode (dkv_append_decode_attn): every
stored field (codes, scales, keyframes, reconstruction state), the lengths and
the attention output equal those of the separate calls (dkv_append, then
dkv_decode_attn / dkv_decode_attn_mq) step after step, and the stored fields
equal the oracle's encoding of the whole sequences.  Covered: one and several
new tokens per sequence, steps across keyframe boundaries, kf below, at and
above 32, ragged and empty sequences, more than 8 virtual heads per kv head
(tokens re-written by each head group), a paged cache, the two exposed
halves, and a sequence whose tokens do not fit."""
import numpy as np
import pytest
import torch

import synthetic as S
from _parity import ATTN_TOL, export_np, oracle_fields, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCALE = 0.088


def _tokens(X, lens, n):
    """[B, Hkv, n, D]: for every batch entry the n tokens after its length."""
    return torch.stack([X[b, :, lens[b]:lens[b] + n] for b in range(X.shape[0])]).contiguous()


def _queries(w, n, step, seed=5):
    g = torch.Generator().manual_seed(seed + 1000 * step)
    shape = (w.B, w.Hq, w.D) if n == 1 else (w.B, n, w.Hq, w.D)
    return torch.randn(shape, generator=g).to(w.q_dtype)


def _check_fields_against_oracle(orc, cache, K, V, lens, kf, cap):
    ex = export_np(cache)
    for b in range(K.shape[0]):
        for h in range(K.shape[1]):
            for t, X in enumerate((K, V)):
                ref = oracle_fields(orc, "delta", X[b, h, :lens[b]].float().numpy(), kf, cap)
                for k in ("codes", "scales"):
                    assert np.array_equal(ex[k][b, h, t], ref[k]), (b, h, t, k)
                nkf = ref["keyframes"].shape[0]
                assert np.array_equal(ex["keyframes"][b, h, t][:nkf], ref["keyframes"])
                if lens[b] > 0:
                    assert np.array_equal(ex["state"][b, h, t].view(np.uint32),
                                          ref["state"].view(np.uint32)), (b, h, t)


def _run_pair(dkv_gpu, w, K, V, lens0, n, steps, kf, cap, paged_pg=0, halves=False):
    """Two caches fed the same tokens: one by the separate calls, one by the
    fused call; returns them with the final lengths after checking every step."""
    sl = torch.tensor(lens0, dtype=torch.int32, device=DEV)
    if paged_pg:
        n_groups = -(-cap // kf)
        max_pages = -(-n_groups // paged_pg)
        n_pages = w.B * max_pages + 3
        g = torch.Generator().manual_seed(9)
        bt = torch.randperm(n_pages, generator=g)[:w.B * max_pages].view(w.B, max_pages)
        fused = dkv_gpu.Cache(w.B, w.Hkv, cap, "delta", kf=kf, page_groups=paged_pg,
                              n_pages=n_pages, block_table=bt.to(torch.int32))
    else:
        fused = dkv_gpu.Cache(w.B, w.Hkv, cap, "delta", kf=kf)
    sep = dkv_gpu.Cache(w.B, w.Hkv, cap, "delta", kf=kf)
    Kd, Vd = K.to(DEV), V.to(DEV)
    T0 = max(lens0)
    for c in (sep, fused):
        c.encode(Kd[:, :, :T0].contiguous(), Vd[:, :, :T0].contiguous(), seq_lens=sl)
    lens = list(lens0)
    for s in range(steps):
        Kn, Vn = _tokens(Kd, lens, n), _tokens(Vd, lens, n)
        q = _queries(w, n, s).to(DEV)
        sep.append(Kn, Vn)
        ref = sep.decode_attn(q, SCALE) if n == 1 else sep.decode_attn_mq(q, SCALE)
        if halves:
            ws = fused.workspace_mq(w.Hq, n)
            got = torch.empty(q.shape, dtype=torch.float32, device=DEV)
            dkv_gpu.dkv_append_decode_attn_split(fused.c, Kn, Vn, dkv_gpu._dtype_code(Kn.dtype), n,
                                                 q, dkv_gpu._dtype_code(q.dtype), w.Hq, SCALE, ws,
                                                 ws.numel() * 4)
            dkv_gpu.dkv_append_decode_attn_merge(fused.c, n, w.Hq, got, ws, ws.numel() * 4)
        else:
            got = fused.append_decode_attn(Kn, Vn, q, SCALE)
        torch.cuda.synchronize()
        assert sep.device_status() == 0 and fused.device_status() == 0, s
        lens = [L + n for L in lens]
        assert fused.seq_lens().tolist() == lens == sep.seq_lens().tolist(), s
        err = row_rel_err(got.cpu().numpy(), ref.cpu().numpy()).max()
        assert err <= 1e-6, (s, err)
    a, b = export_np(sep), export_np(fused)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    return sep, fused, lens


@pytest.mark.parametrize("name,kf,lens0,steps", [
    ("llama3_8b_layer", 32, [60, 0, 31], 40),      # crosses positions 32 and 64; empty entry
    ("llama3_8b_layer", 16, [5, 17, 0], 24),       # kf < 32: tail-zeroed groups
    ("llama3_8b_layer", 64, [60, 1, 127], 12),     # kf > 32: segmented groups
    ("llama3_70b_layer", 32, [95, 33], 6),         # G = 8
])
def test_fused_one_token_equals_separate_calls(orc, dkv_gpu, name, kf, lens0, steps):
    w = S.WORKLOADS[name].with_(B=len(lens0), T=max(lens0) + steps + 1, kf=kf)
    K, V = S.gen_kv(w)
    cap = w.T + 3
    _, fused, lens = _run_pair(dkv_gpu, w, K, V, lens0, 1, steps, kf, cap)
    _check_fields_against_oracle(orc, fused, K, V, lens, kf, cap)


@pytest.mark.parametrize("name,n,kf", [("llama3_8b_layer", 3, 32),   # 12 virtual heads: 2 groups
                                       ("llama3_8b_layer", 2, 16),
                                       ("llama3_70b_layer", 2, 64)])
def test_fused_several_tokens_equals_separate_calls(orc, dkv_gpu, name, n, kf):
    lens0 = [30, 0, 61]
    steps = 5
    w = S.WORKLOADS[name].with_(B=3, T=max(lens0) + n * steps + 1, kf=kf)
    K, V = S.gen_kv(w)
    cap = w.T + 2
    _, fused, lens = _run_pair(dkv_gpu, w, K, V, lens0, n, steps, kf, cap)
    _check_fields_against_oracle(orc, fused, K, V, lens, kf, cap)


def test_fused_attention_matches_oracle(orc, dkv_gpu):
    """The fused call's output against the oracle's attention over the grown
    sequences (not only against the separate calls)."""
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, T=700, kf=32)
    K, V = S.gen_kv(w)
    lens0 = [639, 400]
    cache = dkv_gpu.Cache(w.B, w.Hkv, 704, "delta", kf=32)
    sl = torch.tensor(lens0, dtype=torch.int32, device=DEV)
    cache.encode(K[:, :, :639].contiguous().to(DEV), V[:, :, :639].contiguous().to(DEV),
                 seq_lens=sl)
    Kn, Vn = _tokens(K, lens0, 1).to(DEV), _tokens(V, lens0, 1).to(DEV)
    q = _queries(w, 1, 0)
    out = cache.append_decode_attn(Kn, Vn, q.to(DEV), SCALE)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    G = w.Hq // w.Hkv
    got = out.cpu().numpy()
    for b, L in enumerate(lens0):
        for h in range(w.Hkv):
            ref = orc.decode_attention("delta", q[b, h * G:(h + 1) * G].double().numpy()[None],
                                       K[b:b + 1, h:h + 1, :L + 1].float().numpy(),
                                       V[b:b + 1, h:h + 1, :L + 1].float().numpy(),
                                       kf=32, scale=SCALE)[0]
            err = row_rel_err(got[b, h * G:(h + 1) * G], ref).max()
            assert err <= ATTN_TOL, (b, h, err)


def test_fused_paged_and_halves(orc, dkv_gpu):
    """Through a block table over a shuffled pool (pages of 3 groups), driven
    by the two exposed launches."""
    lens0 = [90, 7]
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, T=130, kf=32)
    K, V = S.gen_kv(w)
    _, fused, lens = _run_pair(dkv_gpu, w, K, V, lens0, 1, 20, 32, 160, paged_pg=3, halves=True)
    _check_fields_against_oracle(orc, fused, K, V, lens, 32, 160)


def test_fused_capacity_entry_keeps_its_length_and_state(dkv_gpu):
    """An entry that is full takes no token (DKV_DEV_CAPACITY) and is decoded
    at its stored length; the others advance; all match the separate calls."""
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=3, T=70, kf=32)
    K, V = S.gen_kv(w)
    cap = 64
    lens0 = [64, 10, 63]
    sl = torch.tensor(lens0, dtype=torch.int32, device=DEV)
    caches = [dkv_gpu.Cache(w.B, w.Hkv, cap, "delta", kf=32) for _ in range(2)]
    Kd, Vd = K.to(DEV), V.to(DEV)
    for c in caches:
        c.encode(Kd[:, :, :64].contiguous(), Vd[:, :, :64].contiguous(), seq_lens=sl)
    # token index per entry clamped so the gather stays inside the arrays
    Kn = _tokens(Kd, [min(L, 63) for L in lens0], 1)
    Vn = _tokens(Vd, [min(L, 63) for L in lens0], 1)
    q = _queries(w, 1, 0).to(DEV)
    sep, fused = caches
    sep.append(Kn, Vn)
    ref = sep.decode_attn(q, SCALE)
    got = fused.append_decode_attn(Kn, Vn, q, SCALE)
    torch.cuda.synchronize()
    for c in caches:
        assert c.device_status() & dkv_gpu.DEV_CAPACITY
        assert c.seq_lens().tolist() == [64, 11, 64]
    assert row_rel_err(got.cpu().numpy(), ref.cpu().numpy()).max() <= 1e-6
    a, b = export_np(sep), export_np(fused)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
