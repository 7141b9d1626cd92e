"""GPU parity of the long-range reference encoder (dkv_lr_encode, the
training-free part of DeltaKV): the chosen references, the fp16 reference
values, the scales, the codes and the reconstruction equal the CPU oracle's
bit for bit, over strides, reference counts (including ties from exact
repeats), input dtypes and ragged lengths; and on the window-repeat
generator the residual against the references is far smaller than plain
Q4_0's error (the long-range similarity the page describes)."""
import numpy as np
import pytest
import torch

import synthetic as S
from _parity import ATTN_TOL, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check(orc, X, s, m, got):
    for q in range(X.shape[0]):
        ref = orc.lr_encode(X[q].float().numpy(), s, m)
        assert np.array_equal(got["ref"][q].cpu().numpy(), ref["ref"]), (q, s, m)
        assert np.array_equal(got["ref_values"][q].cpu().numpy().view(np.uint16), ref["kfr"])
        assert np.array_equal(got["scales"][q].cpu().numpy().view(np.uint16), ref["scales"])
        assert np.array_equal(got["codes"][q].cpu().numpy(), ref["codes"])
        assert np.array_equal(got["xhat"][q].cpu().numpy().view(np.uint32),
                              ref["xhat"].view(np.uint32))


@pytest.mark.parametrize("T,s,m", [(300, 8, 1), (517, 32, 4), (200, 3, 8), (64, 1, 2),
                                   (97, 128, 3)])
def test_lr_encode_bit_exact(orc, dkv_gpu, T, s, m):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=1, Hkv=3, T=T)
    K, _ = S.gen_kv(w)
    X = K[0].contiguous()                       # [3, T, 128] fp16
    X[1, 5::7] = X[1, 0]                        # exact repeats: distance ties
    got = dkv_gpu.lr_encode(X.to(DEV), s, m)
    torch.cuda.synchronize()
    _check(orc, X, s, m, got)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_lr_encode_input_dtypes(orc, dkv_gpu, dtype):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=1, Hkv=2, T=160, kv_dtype=dtype)
    K, _ = S.gen_kv(w)
    X = K[0].contiguous()
    got = dkv_gpu.lr_encode(X.to(DEV), 16, 2)
    torch.cuda.synchronize()
    _check(orc, X, 16, 2, got)


def test_lr_residual_on_window_repeats(orc, dkv_gpu):
    """Window-repeat data (windows copied from far back): with references at
    stride 32 the reconstruction error is a small fraction of plain Q4_0's."""
    w = S.WORKLOADS["batched_decode"].with_(B=1, T=2048, gen="repeat")
    K, V = S.gen_kv(w)
    X = torch.cat([K[0], V[0]]).contiguous()    # [2 Hkv, T, 128]
    got = dkv_gpu.lr_encode(X.to(DEV), 32, 1)
    torch.cuda.synchronize()
    x = X.float().numpy()
    lr = ((got["xhat"].cpu().numpy() - x) ** 2).sum()
    q4 = sum(((orc.q4_encode(x[i])[2] - x[i]) ** 2).sum() for i in range(x.shape[0]))
    print(f"[lr] window-repeat rel error: long-range refs {lr / (x ** 2).sum():.3e}, "
          f"Q4_0 {q4 / (x ** 2).sum():.3e}")
    assert lr < 0.5 * q4


# ---------------------------------------------------------------------------
# decode attention over the long-range reference encoding (dkv_lr_decode_attn)
# ---------------------------------------------------------------------------
def _lr_decode_case(orc, dkv, w, s, m, lens, qdtype, scale):
    """Encode K and V of every (batch entry, kv head) on the GPU, decode, and
    compare with the oracle's binary64 attention over its own reconstruction
    of each prefix (the encoding is causal: a prefix's encoding is the prefix
    of the encoding)."""
    K, V = S.gen_kv(w)
    B, Hkv, T = w.B, w.Hkv, w.T
    G = w.Hq // Hkv
    Xk = K.reshape(B * Hkv, T, 128).contiguous()
    Xv = V.reshape(B * Hkv, T, 128).contiguous()
    ek = dkv.lr_encode(Xk.to(DEV), s, m)
    ev = dkv.lr_encode(Xv.to(DEV), s, m)
    g = torch.Generator().manual_seed(11 * s + m)
    q = torch.randn((B, w.Hq, 128), generator=g).to(qdtype)
    ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out = dkv.lr_decode_attn(ek, ev, q.to(DEV), scale, s, Hkv, lens=ln)
    torch.cuda.synchronize()
    got = out.cpu().double().numpy()
    qd = q.double().numpy()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            L = lens[b]
            rows = got[b, h * G:(h + 1) * G]
            if L == 0:
                assert (rows == 0).all()
                continue
            kh = orc.encode_cache("lr", Xk[b * Hkv + h, :L].float().numpy(), s, n_refs=m)["xhat"]
            vh = orc.encode_cache("lr", Xv[b * Hkv + h, :L].float().numpy(), s, n_refs=m)["xhat"]
            ref = orc.attn(qd[b, h * G:(h + 1) * G], kh, vh, scale)
            worst = max(worst, float(row_rel_err(rows, ref).max()))
    return worst


@pytest.mark.parametrize("s,m,G,qdtype", [(32, 1, 8, torch.bfloat16), (32, 4, 4, torch.float16),
                                          (7, 2, 8, torch.float32), (128, 3, 1, torch.bfloat16)])
def test_lr_decode_matches_oracle(orc, dkv_gpu, s, m, G, qdtype):
    w = S.WORKLOADS["batched_decode"].with_(B=3, Hkv=2, Hq=2 * G, T=700, gen="repeat")
    err = _lr_decode_case(orc, dkv_gpu, w, s, m, [700, 389, 33], qdtype, 1.0 / np.sqrt(128))
    print(f"[lr-decode] s={s} m={m} G={G} q={qdtype} max_row_rel_err={err:.3e}")
    assert err <= ATTN_TOL, err


def test_lr_decode_stride_1_is_the_fp16_cache(orc, dkv_gpu):
    """Stride 1: every token is a reference held in fp16, so the decode must
    equal attention over the fp16 cache (the oracle's fp16 comparator)."""
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, Hkv=2, Hq=8, T=300)
    K, V = S.gen_kv(w)
    lens = [300, 120]
    Xk = K.reshape(4, 300, 128).contiguous()
    Xv = V.reshape(4, 300, 128).contiguous()
    ek = dkv_gpu.lr_encode(Xk.to(DEV), 1, 2)
    ev = dkv_gpu.lr_encode(Xv.to(DEV), 1, 2)
    q = S.gen_q(w)
    out = dkv_gpu.lr_decode_attn(ek, ev, q.to(DEV), 0.1, 1, 2,
                                 lens=torch.tensor(lens, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    ref = orc.decode_attention("fp16", q.double().numpy(), K.float().numpy(), V.float().numpy(),
                               kf=32, scale=0.1, lengths=lens)
    err = row_rel_err(out.cpu().numpy(), ref).max()
    assert err <= ATTN_TOL, err


def test_lr_decode_stress_and_empty(orc, dkv_gpu):
    """Jumpy data, a large softmax scale, lengths 0, 1 and one reference."""
    w = S.WORKLOADS["llama3_70b_layer"].with_(B=4, Hkv=1, Hq=8, T=260, jump_p=0.1)
    err = _lr_decode_case(orc, dkv_gpu, w, 16, 2, [260, 0, 1, 17], torch.bfloat16, 0.5)
    assert err <= ATTN_TOL, err
