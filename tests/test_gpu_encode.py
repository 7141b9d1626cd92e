"""GPU parity of the encoders: codes, scales, keyframes and the closed-loop
state exported from the CUDA cache must equal the CPU oracle bit for bit."""
import numpy as np
import pytest
import torch

import synthetic as S
from _parity import export_np, oracle_fields

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_fields(orc, cache, fmt, K, V, lens, kf, cap):
    ex = export_np(cache)
    B, H = K.shape[0], K.shape[1]
    for b in range(B):
        for h in range(H):
            for t, X in enumerate((K, V)):
                ref = oracle_fields(orc, fmt, X[b, h, :lens[b]].float().numpy(), kf, cap)
                for k, r in ref.items():
                    got = ex[k][b, h, t]
                    if k == "keyframes" and fmt == "delta":
                        got = got[: r.shape[0]]
                    if k == "state":
                        if lens[b] == 0:
                            continue
                        assert np.array_equal(got.view(np.uint32), r.view(np.uint32)), (b, h, t, k)
                    else:
                        bad = np.argwhere(got != r)
                        assert bad.size == 0, (fmt, b, h, t, k, bad[:3].tolist())


@pytest.mark.parametrize("fmt", ["delta", "q4", "fp16"])
@pytest.mark.parametrize("kf", [1, 2, 32, 33, 512])
def test_encode_bit_exact(orc, dkv_gpu, fmt, kf):
    if fmt != "delta" and kf != 32:
        pytest.skip("kf only matters for the delta format")
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, Hkv=2, T=600)
    K, V = S.gen_kv(w)
    lens = [600, 437]
    cap = 640
    cache = dkv_gpu.Cache(2, 2, cap, fmt, kf=kf)
    seq = torch.tensor(lens, dtype=torch.int32, device=DEV)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=seq)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == lens
    _check_fields(orc, cache, fmt, K, V, lens, kf, cap)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_encode_input_dtypes(orc, dkv_gpu, dtype):
    w = S.WORKLOADS["tiny"].with_(B=1, Hkv=1, T=300, kv_dtype=dtype)
    K, V = S.gen_kv(w)
    cache = dkv_gpu.Cache(1, 1, 300, "delta", kf=32)
    cache.encode(K.to(DEV), V.to(DEV))
    torch.cuda.synchronize()
    _check_fields(orc, cache, "delta", K, V, [300], 32, 300)


@pytest.mark.parametrize("fmt", ["delta", "q4", "fp16"])
@pytest.mark.parametrize("kf", [2, 32, 33])
def test_append_continues_closed_loop(orc, dkv_gpu, fmt, kf):
    if fmt != "delta" and kf != 32:
        pytest.skip("kf only matters for the delta format")
    w = S.WORKLOADS["ragged_long"].with_(B=2, Hkv=2, T=400, ragged=None)
    K, V = S.gen_kv(w)
    cap = 420
    cache = dkv_gpu.Cache(2, 2, cap, fmt, kf=kf)
    T0 = 97
    cache.encode(K[:, :, :T0].contiguous().to(DEV), V[:, :, :T0].contiguous().to(DEV))
    pos = T0
    for n in (1, 1, 5, 31, 32, 33, 64, 1, 135):
        cache.append(K[:, :, pos:pos + n].contiguous().to(DEV), V[:, :, pos:pos + n].contiguous().to(DEV))
        pos += n
    torch.cuda.synchronize()
    assert pos == 400
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == [400, 400]
    _check_fields(orc, cache, fmt, K, V, [400, 400], kf, cap)


def test_append_past_capacity_sets_status(dkv_gpu):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, Hkv=1, T=40)
    K, V = S.gen_kv(w)
    cache = dkv_gpu.Cache(2, 1, 40, "delta", kf=32)
    seq = torch.tensor([30, 38], dtype=torch.int32, device=DEV)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=seq)
    cache.append(K[:, :, :3].contiguous().to(DEV), V[:, :, :3].contiguous().to(DEV))
    torch.cuda.synchronize()
    st = cache.device_status()
    assert st & dkv_gpu.DEV_CAPACITY
    assert cache.seq_lens().tolist() == [33, 38]      # entry 1 skipped, entry 0 appended
    assert cache.device_status() == 0                 # cleared by the read


def test_encode_bad_lengths_set_status(dkv_gpu):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, Hkv=1, T=40)
    K, V = S.gen_kv(w)
    cache = dkv_gpu.Cache(2, 1, 40, "delta", kf=32)
    seq = torch.tensor([41, 10], dtype=torch.int32, device=DEV)   # 41 > T
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=seq)
    torch.cuda.synchronize()
    assert cache.device_status() & dkv_gpu.DEV_BAD_SEQLEN
    assert cache.seq_lens().tolist() == [0, 10]


def test_dequantize_matches_oracle_reconstruction(orc, dkv_gpu):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=1, Hkv=2, T=300)
    K, V = S.gen_kv(w)
    for fmt in ("delta", "q4", "fp16"):
        cache = dkv_gpu.Cache(1, 2, 300, fmt, kf=32)
        cache.encode(K.to(DEV), V.to(DEV))
        xh = cache.dequantize().cpu().numpy()
        for h in range(2):
            for t, X in enumerate((K, V)):
                ref = orc.encode_cache(fmt, X[0, h].float().numpy(), 32)["xhat"]
                assert np.array_equal(xh[0, h, t].view(np.uint32), ref.view(np.uint32)), (fmt, h, t)


def test_encoder_quotient_is_ieee_division(dkv_gpu):
    """The delta encoder divides each delta by the block scale with one
    correctly rounded reciprocal and Markstein's correction; it must give the
    IEEE quotient bit for bit wherever that quotient is a normal number, and
    the same code everywhere (a subnormal quotient, which needs a subnormal
    delta, always gives code 8).  Checked for every finite non-zero fp16 scale
    b and dividends RN(u b) (and their neighbours, including the smallest
    subnormals next to an underflowed 0) with u over the quotients the block
    rule meets: dense in [-17, 17], the exact halves k + 1/2, and small powers
    of two down to 2^-60."""
    g = torch.Generator().manual_seed(0)
    u = torch.cat([torch.linspace(-17.0, 17.0, 24001, dtype=torch.float64),
                   torch.arange(-34, 35, dtype=torch.float64) / 2.0,
                   torch.rand(8000, generator=g, dtype=torch.float64) * 34.0 - 17.0,
                   torch.tensor([s * 2.0 ** -k for k in range(1, 61) for s in (1, -1)],
                                dtype=torch.float64)]).float().to(DEV)
    bad = torch.zeros(2, dtype=torch.int64, device=DEV)
    dkv_gpu.dkv_debug_division_check(u, bad)
    torch.cuda.synchronize()
    assert bad[0].item() == 0, bad[0].item()
