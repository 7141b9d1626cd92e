"""GPU parity of the paged cache (delta format): records reached through a
caller-owned block table over a shuffled page pool give the oracle's stored
fields bit for bit and its attention within the tolerance, including odd page
sizes (stages split at page boundaries), kf > 32, ragged lengths, appends that
cross pages, and a bad block-table entry that is flagged, not followed."""
import numpy as np
import pytest
import torch

import synthetic as S
from _parity import ATTN_TOL, export_np, oracle_fields, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _paged(dkv_gpu, B, H, cap, kf, pg, extra_pages=5, seed=3):
    n_groups = -(-cap // kf)
    max_pages = -(-n_groups // pg)
    n_pages = B * max_pages + extra_pages
    g = torch.Generator().manual_seed(seed)
    bt = torch.randperm(n_pages, generator=g)[:B * max_pages].view(B, max_pages).to(torch.int32)
    return dkv_gpu.Cache(B, H, cap, "delta", kf=kf, page_groups=pg, n_pages=n_pages,
                         block_table=bt)


@pytest.mark.parametrize("kf,pg", [(32, 1), (32, 3), (32, 16), (16, 5), (64, 2)])
def test_paged_encode_and_decode(orc, dkv_gpu, kf, pg):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=3, T=1500)
    K, V = S.gen_kv(w)
    lens = [1500, 0, 777]
    cap = 1536
    cache = _paged(dkv_gpu, w.B, w.Hkv, cap, kf, pg)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV))
    q = S.gen_q(w)
    out = cache.decode_attn(q.to(DEV), 0.088)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    ex = export_np(cache)
    for b in range(w.B):
        for h in range(w.Hkv):
            for t, X in enumerate((K, V)):
                ref = oracle_fields(orc, "delta", X[b, h, :lens[b]].float().numpy(), kf, cap)
                for k in ("codes", "scales"):
                    assert np.array_equal(ex[k][b, h, t], ref[k]), (kf, pg, b, h, t, k)
                nkf = ref["keyframes"].shape[0]
                assert np.array_equal(ex["keyframes"][b, h, t][:nkf], ref["keyframes"])
    G = w.Hq // w.Hkv
    for b in range(w.B):
        got = out[b].cpu().numpy()
        if lens[b] == 0:
            assert not got.any()
            continue
        for h in range(w.Hkv):
            ref = orc.decode_attention("delta", q[b, h * G:(h + 1) * G].double().numpy()[None],
                                       K[b:b + 1, h:h + 1, :lens[b]].float().numpy(),
                                       V[b:b + 1, h:h + 1, :lens[b]].float().numpy(),
                                       kf=kf, scale=0.088)[0]
            err = row_rel_err(got[h * G:(h + 1) * G], ref).max()
            assert err <= ATTN_TOL, (kf, pg, b, h, err)


def test_paged_appends_cross_pages(orc, dkv_gpu):
    """Single-token appends over several page boundaries (one group per page)
    give the same stored fields as a contiguous cache fed the same tokens."""
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, T=300)
    K, V = S.gen_kv(w)
    cap, kf = 320, 32
    paged = _paged(dkv_gpu, w.B, w.Hkv, cap, kf, 1)
    flat = dkv_gpu.Cache(w.B, w.Hkv, cap, "delta", kf=kf)
    T0 = 200
    for c in (paged, flat):
        c.encode(K[:, :, :T0].contiguous().to(DEV), V[:, :, :T0].contiguous().to(DEV))
        for p in range(T0, w.T):
            c.append(K[:, :, p:p + 1].contiguous().to(DEV), V[:, :, p:p + 1].contiguous().to(DEV))
    torch.cuda.synchronize()
    assert paged.device_status() == 0 and flat.device_status() == 0
    assert paged.seq_lens().tolist() == [w.T] * w.B
    a, b = export_np(paged), export_np(flat)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    q = S.gen_q(w).to(DEV)
    o1, o2 = paged.decode_attn(q, 0.088), flat.decode_attn(q, 0.088)
    torch.cuda.synchronize()
    assert row_rel_err(o1.cpu().numpy(), o2.cpu().numpy()).max() <= 1e-6


def test_paged_bad_block_table_entry_is_flagged(dkv_gpu):
    """An entry outside the pool sets DKV_DEV_BAD_PAGE and the call returns
    (nothing is read or written through it); with the entry restored the
    same cache decodes as before."""
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=1, T=256)
    K, V = S.gen_kv(w)
    cache = _paged(dkv_gpu, 1, w.Hkv, 256, 32, 2)
    cache.encode(K.to(DEV), V.to(DEV))
    q = S.gen_q(w).to(DEV)
    ref = cache.decode_attn(q, 0.088).clone()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    good = int(cache.block_table[0, 1])
    cache.block_table[0, 1] = cache.c.n_pages + 7
    cache.decode_attn(q, 0.088)
    torch.cuda.synchronize()
    assert cache.device_status() & dkv_gpu.DEV_BAD_PAGE
    cache.block_table[0, 1] = good
    again = cache.decode_attn(q, 0.088)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert torch.equal(again, ref)
