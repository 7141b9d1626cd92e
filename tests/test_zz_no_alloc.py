"""dkv_decode_attn_noalloc: the decode step for callers that cannot allocate
device memory when they decode (graph capture, engines that pre-plan every
allocation).  Called through the C ABI, its output must equal the regular
dkv_decode_attn (which takes a caller-allocated workspace) bit for bit: both
run the same kernels on the same grid, only the scratch address differs.
Checked on two calls in a row, after a differently shaped call has left its
partial records in the library's shared scratch array (a stale record read by
mistake would show).

The file name sorts last so that a run stopping at the first failure has
already run every other test."""
import math

import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _stale_call(dkv):
    """A decode through the no-workspace entry point on another shape, so the
    shared array holds records that are not the next call's."""
    w = S.WORKLOADS["llama3_8b_layer"].with_(B=5, Hkv=2, Hq=16, T=1300, kf=32)
    K, V = S.gen_kv(w)
    cache = dkv.Cache(w.B, w.Hkv, w.T, "delta", kf=32)
    cache.encode(K.to(DEV), V.to(DEV))
    q = (S.gen_q(w) * 4).to(DEV)
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=DEV)
    dkv.dkv_decode_attn_noalloc(cache.c, q, dkv.DKV_F16, w.Hq, 0.3, out)
    torch.cuda.synchronize()


@pytest.mark.parametrize("fmt,kf", [("delta", 32), ("delta", 512), ("q4", 32)])
def test_noalloc_matches_workspace_entry_point(dkv_gpu, fmt, kf):
    dkv = dkv_gpu
    _stale_call(dkv)
    w = S.WORKLOADS["llama3_70b_layer"].with_(B=3, Hkv=4, Hq=32, T=900, kf=kf)
    K, V = S.gen_kv(w)
    cache = dkv.Cache(w.B, w.Hkv, w.T, fmt, kf=kf)
    cache.encode(K.to(DEV), V.to(DEV))
    scale = 1.0 / math.sqrt(128)
    qcode = dkv.DKV_BF16
    for call in range(2):
        q = S.gen_q(w, step=call).to(DEV)
        ref = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=DEV)
        ws = cache.workspace(w.Hq)
        dkv.dkv_decode_attn(cache.c, q, qcode, w.Hq, scale, ref, ws, ws.numel() * 4)
        got = torch.full_like(ref, float("nan"))
        dkv.dkv_decode_attn_noalloc(cache.c, q, qcode, w.Hq, scale, got)
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        assert torch.equal(got, ref), (call, (got - ref).abs().max().item())


def test_noalloc_rejects_oversized_steps(dkv_gpu):
    dkv = dkv_gpu
    # enough sequences that the partial records exceed the 16 MiB array
    cache = dkv.Cache(1024, 8, 32, "delta", kf=32)
    q = torch.zeros((1024, 512, 128), dtype=torch.float16, device=DEV)
    out = torch.empty((1024, 512, 128), dtype=torch.float32, device=DEV)
    need = dkv.dkv_decode_workspace_bytes(cache.desc, 512)
    assert need > (16 << 20)
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_decode_attn_noalloc(cache.c, q, dkv.DKV_F16, 512, 1.0, out)
    assert e.value.status == dkv.DKV_ECAPACITY
