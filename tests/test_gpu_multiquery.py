"""GPU parity of multi-query decode (several new tokens per sequence, as in
speculative decoding): query t of a sequence of length L attends to the
positions before L - (nq - 1 - t), against the CPU oracle over exactly that
prefix; nq = 1 equals the one-query entry point bit for bit."""
import numpy as np
import pytest
import torch

import synthetic as S
from _parity import ATTN_TOL, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,nq,kf", [("llama3_8b_layer", 1, 32), ("llama3_8b_layer", 2, 32),
                                        ("llama3_8b_layer", 3, 64),
                                        ("llama3_70b_layer", 2, 32)])
def test_multiquery_matches_oracle(orc, dkv_gpu, name, nq, kf):
    w = S.WORKLOADS[name].with_(B=3, T=900, kf=kf)
    K, V = S.gen_kv(w)
    lens = [900, 2, 555]                         # entry 1: shorter than the queries for nq = 3
    cache = dkv_gpu.Cache(w.B, w.Hkv, w.T, "delta", kf=kf)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV))
    g = torch.Generator().manual_seed(11 + nq)
    Q = torch.randn((w.B, nq, w.Hq, w.D), generator=g).to(w.q_dtype)
    scale = 0.088
    out = cache.decode_attn_mq(Q.to(DEV), scale)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    got = out.cpu().numpy()
    for b in range(w.B):
        for t in range(nq):
            L = lens[b] - (nq - 1 - t)
            if L <= 0:
                assert not got[b, t].any()
                continue
            ref = orc.decode_attention("delta", Q[b:b + 1, t].double().numpy(),
                                       K[b:b + 1, :, :L].float().numpy(),
                                       V[b:b + 1, :, :L].float().numpy(), kf=kf, scale=scale)[0]
            err = row_rel_err(got[b, t], ref).max()
            print(f"[multiquery] {name} nq={nq} kf={kf} b={b} t={t} L={L} max_row_rel_err={err:.3e}")
            assert err <= ATTN_TOL, (b, t, err)


def test_single_query_equals_decode_attn(dkv_gpu):
    w = S.WORKLOADS["llama3_70b_layer"].with_(B=2, T=700)
    K, V = S.gen_kv(w)
    cache = dkv_gpu.Cache(w.B, w.Hkv, w.T, "delta", kf=32)
    cache.encode(K.to(DEV), V.to(DEV))
    q = S.gen_q(w).to(DEV)
    a = cache.decode_attn(q, 0.088)
    b = cache.decode_attn_mq(q[:, None].contiguous(), 0.088)[:, 0]
    torch.cuda.synchronize()
    assert torch.equal(a, b)
