"""GPU parity of dkv_decode_attn against the CPU oracle (binary64 softmax
attention over the oracle's own reconstruction), within the row-relative
tolerance 2e-3 (fp32 accumulation)."""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from _parity import ATTN_TOL, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(orc, dkv, w, fmt, lens=None, cap=None, scale=None):
    K, V = S.gen_kv(w)
    q = S.gen_q(w)
    lens = lens or [w.T] * w.B
    cap = cap or w.T
    scale = scale if scale is not None else 1.0 / math.sqrt(128)
    cache = dkv.Cache(w.B, w.Hkv, cap, fmt, kf=w.kf)
    seq = torch.tensor(lens, dtype=torch.int32, device=DEV)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=seq)
    out = cache.decode_attn(q.to(DEV), scale)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    ref = orc.decode_attention(fmt, q.double().numpy(), K.float().numpy(), V.float().numpy(),
                               kf=w.kf, scale=scale, lengths=lens)
    got = out.cpu().double().numpy()
    err = row_rel_err(got, ref)
    empty = np.array(lens) == 0
    if empty.any():
        assert (got[empty] == 0).all()
    e = err[~empty].max() if (~empty).any() else 0.0
    print(f"[parity] {w.name} fmt={fmt} kf={w.kf} B={w.B} Hq={w.Hq} Hkv={w.Hkv} T={w.T} "
          f"max_row_rel_err={e:.3e}")
    return e


def test_tiny_fp32(orc, dkv_gpu):
    err = _run(orc, dkv_gpu, S.WORKLOADS["tiny"], "delta")
    assert err <= ATTN_TOL, err


@pytest.mark.parametrize("fmt", ["delta", "q4", "fp16"])
def test_llama3_8b_layer_shape(orc, dkv_gpu, fmt):
    w = S.WORKLOADS["llama3_8b_layer"].with_(T=1000)
    err = _run(orc, dkv_gpu, w, fmt)
    assert err <= ATTN_TOL, err


@pytest.mark.parametrize("fmt", ["delta", "q4", "fp16"])
def test_llama3_70b_layer_shape(orc, dkv_gpu, fmt):
    w = S.WORKLOADS["llama3_70b_layer"].with_(B=2, T=777)
    err = _run(orc, dkv_gpu, w, fmt)
    assert err <= ATTN_TOL, err


@pytest.mark.parametrize("kf", [1, 2, 16, 32, 33, 64, 100, 512])
def test_keyframe_intervals(orc, dkv_gpu, kf):
    w = S.WORKLOADS["llama3_70b_layer"].with_(B=2, Hkv=2, Hq=16, T=1100, kf=kf)
    err = _run(orc, dkv_gpu, w, "delta", lens=[1100, 611])
    assert err <= ATTN_TOL, (kf, err)


@pytest.mark.parametrize("G", [1, 3, 4, 8, 16])
def test_gqa_group_sizes(orc, dkv_gpu, G):
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, Hkv=2, Hq=2 * G, T=300)
    err = _run(orc, dkv_gpu, w, "delta")
    assert err <= ATTN_TOL, (G, err)


@pytest.mark.parametrize("fmt", ["delta", "q4", "fp16"])
def test_ragged_and_empty_sequences(orc, dkv_gpu, fmt):
    w = S.WORKLOADS["ragged_long"].with_(B=5, Hkv=2, Hq=8, T=700, ragged=None)
    err = _run(orc, dkv_gpu, w, fmt, lens=[700, 0, 1, 33, 64], cap=720)
    assert err <= ATTN_TOL, err


@pytest.mark.parametrize("gen", ["repeat", "mixture"])
def test_window_generators(orc, dkv_gpu, gen):
    w = S.WORKLOADS["batched_decode"].with_(B=2, T=640, gen=gen, jump_p=0.0)
    err = _run(orc, dkv_gpu, w, "delta")
    assert err <= ATTN_TOL, err


def test_append_then_decode(orc, dkv_gpu):
    w = S.WORKLOADS["ragged_long"].with_(B=2, Hkv=2, Hq=8, T=300, ragged=None)
    K, V = S.gen_kv(w)
    q = S.gen_q(w)
    cache = dkv_gpu.Cache(2, 2, 300, "delta", kf=32)
    cache.encode(K[:, :, :200].contiguous().to(DEV), V[:, :, :200].contiguous().to(DEV))
    for p in range(200, 300):
        cache.append(K[:, :, p:p + 1].contiguous().to(DEV), V[:, :, p:p + 1].contiguous().to(DEV))
    out = cache.decode_attn(q.to(DEV), 0.125)
    torch.cuda.synchronize()
    ref = orc.decode_attention("delta", q.double().numpy(), K.float().numpy(), V.float().numpy(),
                               kf=32, scale=0.125)
    assert row_rel_err(out.cpu().numpy(), ref).max() <= ATTN_TOL


def test_split_and_merge_entry_points(orc, dkv_gpu):
    w = S.WORKLOADS["llama3_8b_layer"].with_(T=500)
    K, V = S.gen_kv(w)
    q = S.gen_q(w).to(DEV)
    cache = dkv_gpu.Cache(w.B, w.Hkv, w.T, "delta", kf=32)
    cache.encode(K.to(DEV), V.to(DEV))
    a = cache.decode_attn(q, 0.088)
    ws = cache.workspace(w.Hq)
    b = torch.empty_like(a)
    dkv_gpu.dkv_decode_attn_split(cache.c, q, dkv_gpu.DKV_F16, w.Hq, 0.088, ws, ws.numel() * 4)
    dkv_gpu.dkv_decode_attn_merge(cache.c, w.Hq, b, ws, ws.numel() * 4)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_workspace_too_small_is_rejected(dkv_gpu):
    cache = dkv_gpu.Cache(1, 1, 64, "delta", kf=32)
    q = torch.zeros((1, 1, 128), dtype=torch.float16, device=DEV)
    out = torch.empty((1, 1, 128), dtype=torch.float32, device=DEV)
    ws = torch.empty(16, dtype=torch.float32, device=DEV)
    with pytest.raises(dkv_gpu.DkvError) as e:
        dkv_gpu.dkv_decode_attn(cache.c, q, dkv_gpu.DKV_F16, 1, 1.0, out, ws, 64)
    assert e.value.status == dkv_gpu.DKV_ECAPACITY


def test_pipeline_wait_timeout_is_reported_not_hung(dkv_gpu):
    """Failure detection without a GPU fault: with the copies dropped on
    purpose, every bounded wait runs out (~1 s), the kernel records
    DKV_DEV_TIMEOUT and returns; the context stays usable afterwards."""
    import time
    w = S.WORKLOADS["llama3_8b_layer"].with_(T=256)
    K, V = S.gen_kv(w)
    q = S.gen_q(w).to(DEV)
    cache = dkv_gpu.Cache(w.B, w.Hkv, w.T, "delta", kf=32)
    cache.encode(K.to(DEV), V.to(DEV))
    good = cache.decode_attn(q, 0.088).clone()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    dkv_gpu.dkv_debug_set_fault(1)
    try:
        t0 = time.time()
        cache.decode_attn(q, 0.088)
        st = cache.device_status()          # synchronises
        dt = time.time() - t0
    finally:
        dkv_gpu.dkv_debug_set_fault(0)
    assert st & dkv_gpu.DEV_TIMEOUT
    assert dt < 30.0
    again = cache.decode_attn(q, 0.088)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert torch.equal(again, good)
