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
