"""GPU parity on the corner cases of the block rule inside the closed loop.

The token sequences of ``_edge`` make the closed-loop deltas hit, at every kf:
the hand-worked golden blocks, +a/-a ties at low and high lanes in both
orders, exact half-way points (k + 1/2) d, the element at -m (code 15),
all-zero delta blocks (scale bits 0x8000), scales that are fp16 subnormals or
round to zero, rounded subnormal scales below m/8 (codes clamped at 0), large
and random blocks.  A constant fp16 sequence gives all-zero deltas.  The
stored fields written by each of the three CUDA writers -- the encoder
(dkv_encode), the append (dkv_append) and the quantiser inside the fused
append + decode (dkv_append_decode_attn) -- must equal the oracle's encoding
bit for bit; the decode over these sequences must match the oracle's
attention within the row-relative 2e-3.

Source: page "영상 압축 기법을 KV 캐시에 적용해 Q4 양자화 오차를 10,000배 줄인
Delta-KV", section "핵심 아이디어" (keyframe + Q4_0-quantised token deltas).
"""
import math

import numpy as np
import pytest
import torch

import _edge as E
from _parity import ATTN_TOL, assert_fields_equal, row_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
KFS = [1, 2, 32, 33, 512]


def _edge_kv(orc, B, H, T, kf, seed):
    K = np.stack([np.stack([E.edge_sequence(orc, T, kf, seed + 100 * b + 10 * h)
                            for h in range(H)]) for b in range(B)])
    V = np.stack([np.stack([E.edge_sequence(orc, T, kf, seed + 5000 + 100 * b + 10 * h)
                            for h in range(H)]) for b in range(B)])
    return torch.from_numpy(K), torch.from_numpy(V)


def _T(kf):
    return 1100 if kf == 512 else 300


def _assert_covered(orc, K, kf):
    if kf == 1:
        return
    tot = {}
    for b in range(K.shape[0]):
        for h in range(K.shape[1]):
            x = K[b, h].numpy()
            c = E.coverage(x, kf, orc.delta_encode(x, kf))
            for k, v in c.items():
                tot[k] = tot.get(k, 0) + v
    for k in ("tie", "tie_high", "zero_block", "half", "clamp15", "clamp0", "sub_d",
              "zero_d_nonzero"):
        assert tot[k] > 0, (kf, k, tot)


@pytest.mark.parametrize("kf", KFS)
def test_edge_blocks_encode_and_decode(orc, dkv_gpu, kf):
    T = _T(kf)
    K, V = _edge_kv(orc, 2, 2, T, kf, 11 * kf)
    _assert_covered(orc, K, kf)
    lens = [T, T - 77]
    cap = T + 4
    cache = dkv_gpu.Cache(2, 2, cap, "delta", kf=kf)
    cache.encode(K.to(DEV), V.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32,
                                                             device=DEV))
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == lens
    assert_fields_equal(orc, cache, "delta", K, V, lens, kf, cap)
    # the decode over the same cache
    g = torch.Generator().manual_seed(kf)
    q = torch.randn((2, 8, 128), generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(128)
    out = cache.decode_attn(q.to(DEV), scale)
    torch.cuda.synchronize()
    ref = orc.decode_attention("delta", q.double().numpy(), K.numpy(), V.numpy(), kf=kf,
                               scale=scale, lengths=lens)
    err = row_rel_err(out.cpu().numpy(), ref).max()
    print(f"[edge] kf={kf} decode max_row_rel_err={err:.3e}")
    assert err <= ATTN_TOL, err


@pytest.mark.parametrize("kf", KFS)
def test_edge_blocks_append(orc, dkv_gpu, kf):
    T = _T(kf)
    K, V = _edge_kv(orc, 2, 1, T, kf, 13 * kf + 1)
    cap = T
    cache = dkv_gpu.Cache(2, 1, cap, "delta", kf=kf)
    Kd, Vd = K.to(DEV), V.to(DEV)
    pos = 37
    cache.encode(Kd[:, :, :pos].contiguous(), Vd[:, :, :pos].contiguous())
    for n in (1, 2, 31, 32, 33, 64, 1, 3):
        cache.append(Kd[:, :, pos:pos + n].contiguous(), Vd[:, :, pos:pos + n].contiguous())
        pos += n
    cache.append(Kd[:, :, pos:].contiguous(), Vd[:, :, pos:].contiguous())
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == [T, T]
    assert_fields_equal(orc, cache, "delta", K, V, [T, T], kf, cap)


@pytest.mark.parametrize("kf", KFS)
def test_edge_blocks_fused_append(orc, dkv_gpu, kf):
    """The quantiser inside the split kernel: one token per call across
    keyframe boundaries, then calls of three tokens (two head groups of 8
    virtual heads, so every group's warps store the fields)."""
    T = 100 if kf != 512 else 560
    K, V = _edge_kv(orc, 2, 2, T, kf, 17 * kf + 2)
    cap = T
    Hq = 8
    cache = dkv_gpu.Cache(2, 2, cap, "delta", kf=kf)
    Kd, Vd = K.to(DEV), V.to(DEV)
    pos = T - 64
    cache.encode(Kd[:, :, :pos].contiguous(), Vd[:, :, :pos].contiguous())
    g = torch.Generator().manual_seed(3)
    while pos < T:
        n = 1 if pos < T - 30 else min(3, T - pos)
        q = torch.randn((2, Hq, 128) if n == 1 else (2, n, Hq, 128), generator=g)
        cache.append_decode_attn(Kd[:, :, pos:pos + n].contiguous(),
                                 Vd[:, :, pos:pos + n].contiguous(),
                                 q.to(torch.float16).to(DEV), 0.088)
        pos += n
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert cache.seq_lens().tolist() == [T, T]
    assert_fields_equal(orc, cache, "delta", K, V, [T, T], kf, cap)


@pytest.mark.parametrize("kf", KFS)
def test_constant_fp16_sequence(orc, dkv_gpu, kf):
    """A constant fp16 token: every delta is zero, so every delta row stores
    codes 8 and scale bits 0x8000 (fp16(+0 / -8) = -0), through the encoder,
    the append and the fused append."""
    T = 300 if kf != 512 else 700
    x = np.stack([np.stack([E.constant_sequence(T, 31 * b + 7 * h + kf) for h in range(2)])
                  for b in range(2)])
    K = torch.from_numpy(x).to(torch.float16)
    V = torch.from_numpy(x[:, ::-1].copy()).to(torch.float16)
    Kd, Vd = K.to(DEV), V.to(DEV)
    caches = [dkv_gpu.Cache(2, 2, T, "delta", kf=kf) for _ in range(3)]
    caches[0].encode(Kd, Vd)
    half = T // 2
    for c in caches[1:]:
        c.encode(Kd[:, :, :half].contiguous(), Vd[:, :, :half].contiguous())
    caches[1].append(Kd[:, :, half:].contiguous(), Vd[:, :, half:].contiguous())
    for p in range(half, T):
        caches[2].append_decode_attn(Kd[:, :, p:p + 1].contiguous(), Vd[:, :, p:p + 1].contiguous(),
                                     torch.ones((2, 4, 128), dtype=torch.float16, device=DEV), 0.1)
    torch.cuda.synchronize()
    for c in caches:
        assert c.device_status() == 0
        assert_fields_equal(orc, c, "delta", K.float(), V.float(), [T, T], kf, T)
        ex = c.export()
        delta_rows = [p for p in range(T) if p % kf]
        if delta_rows:
            assert (ex["codes"][:, :, :, delta_rows].cpu() == 8).all()
            sc = ex["scales"][:, :, :, delta_rows].cpu().numpy().view(np.uint16)
            assert (sc == 0x8000).all()
