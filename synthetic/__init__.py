"""Seeded synthetic K/V/q generators shared by the tests, the smoke check and
the benchmark.

This module only draws random inputs; it holds none of the method's
arithmetic (no quantiser, no reconstruction, no attention).  Both the CUDA
library and the CPU oracle consume the tensors it returns.

The process per (batch, kv-head, channel c), for K and V independently:

* sigma_c is log-uniform in [0.1, 4];
* x_0 ~ N(0, sigma_c^2);
* random walk x_t = x_{t-1} + N(0, (step * sigma_c)^2), walked in float64 and
  rounded once to the storage dtype (fp16, or fp32 for the tiny case);
* "jump" tokens (probability ``jump_p`` per token) redraw the whole token,
  x_t ~ N(0, sigma_c^2), and the walk continues from there;
* "window repeat" (code-like text): every 64-token window after the first
  copies a uniformly chosen earlier window plus N(0, (0.002 sigma_c)^2) noise;
* "mixture": per 64-token window, walk (0.7), repeat of an earlier window plus
  noise (0.2), or an i.i.d. redraw of every token (0.1).

Queries are N(0, 1) in the query dtype.  Every tensor comes from a
``torch.Generator`` seeded per workload; CPU and CUDA generators give
different (but each reproducible) streams, so a test that needs the same
values on both sides generates on one device and copies.

The workloads mirror the shapes the Delta-KV pages discuss (Llama-3-8B and
Llama-3-70B single layers, batched and ragged long-context decode); no public
dataset is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

WINDOW = 64


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    T: int                      # context per sequence (max for ragged)
    kf: int
    kv_dtype: torch.dtype
    q_dtype: torch.dtype
    gen: str = "walk"           # walk | repeat | mixture
    step: float = 0.01
    jump_p: float = 0.0
    ragged: tuple | None = None  # (lo, hi) for per-sequence lengths
    n_append: int = 0
    seed: int = 1000
    extra: dict = field(default_factory=dict)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # tiny parity case: batch 1, 1 query head / 1 KV head, D 128, context 512
    "tiny": Workload("tiny", 1, 1, 1, 128, 512, 32, torch.float32, torch.float32,
                     "walk", 0.01, 0.0, seed=1000),
    # Llama-3-8B-shaped single layer
    "llama3_8b_layer": Workload("llama3_8b_layer", 1, 32, 8, 128, 4096, 32, torch.float16,
                                torch.float16, "walk", 0.01, 0.01, seed=1001),
    # batched decode, kf 32 (kf 512 and the code-like variant via with_())
    "batched_decode": Workload("batched_decode", 16, 32, 8, 128, 16384, 32, torch.float16,
                               torch.float16, "walk", 0.01, 0.01, seed=1002),
    # Llama-3-70B-shaped single layer: the headline decode workload
    "llama3_70b_layer": Workload("llama3_70b_layer", 16, 64, 8, 128, 32768, 32,
                                 torch.float16, torch.bfloat16, "walk", 0.01, 0.01,
                                 seed=1003),
    # ragged long context with per-token appends
    "ragged_long": Workload("ragged_long", 4, 32, 8, 128, 131072, 32, torch.float16,
                            torch.float16, "mixture", 0.01, 0.0, ragged=(32768, 131072),
                            n_append=256, seed=1004),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _sigma(H: int, D: int, g: torch.Generator, device) -> torch.Tensor:
    u = torch.rand((H, 1, D), generator=g, device=device, dtype=torch.float64)
    return torch.exp(math.log(0.1) + u * (math.log(4.0) - math.log(0.1)))


def _walk(H, T, D, sigma, step, jump_p, g, device):
    """Random walk with whole-token redraws, float64 [H, T, D]."""
    incr = torch.randn((H, T, D), generator=g, device=device, dtype=torch.float64) * (step * sigma)
    cs = torch.cumsum(incr, dim=1)
    fresh = torch.randn((H, T, D), generator=g, device=device, dtype=torch.float64) * sigma
    jumps = torch.rand((H, T), generator=g, device=device) < jump_p
    jumps[:, 0] = True
    t = torch.arange(T, device=device).expand(H, T)
    last = torch.cummax(torch.where(jumps, t, torch.zeros_like(t)), dim=1).values
    idx = last.unsqueeze(-1).expand(H, T, D)
    return torch.gather(fresh, 1, idx) + cs - torch.gather(cs, 1, idx)


def _windows(H, T, D, sigma, step, g, device, p_walk, p_repeat):
    """Window-structured generator (repeat / mixture), float64 [H, T, D]."""
    out = torch.empty((H, T, D), device=device, dtype=torch.float64)
    nwin = (T + WINDOW - 1) // WINDOW
    prev = torch.randn((H, 1, D), generator=g, device=device, dtype=torch.float64) * sigma
    for w in range(nwin):
        a, b = w * WINDOW, min(T, (w + 1) * WINDOW)
        n = b - a
        walk = prev + torch.cumsum(
            torch.randn((H, n, D), generator=g, device=device, dtype=torch.float64)
            * (step * sigma), dim=1)
        if w == 0:
            blk = walk
        else:
            r = torch.rand((H, 1, 1), generator=g, device=device, dtype=torch.float64)
            src = torch.randint(0, w, (H,), generator=g, device=device)
            rows = (src * WINDOW).view(H, 1, 1) + torch.arange(n, device=device).view(1, n, 1)
            rows = rows.clamp(max=a - 1).expand(H, n, D)
            rep = torch.gather(out[:, :a], 1, rows) + torch.randn(
                (H, n, D), generator=g, device=device, dtype=torch.float64) * (0.002 * sigma)
            iid = torch.randn((H, n, D), generator=g, device=device, dtype=torch.float64) * sigma
            blk = torch.where(r < p_walk, walk, torch.where(r < p_walk + p_repeat, rep, iid))
        out[:, a:b] = blk
        prev = blk[:, -1:, :]
    return out


def gen_kv_one(w: Workload, b: int, T: int, device="cpu", seed_offset: int = 0):
    """K and V for batch entry ``b``: two [Hkv, T, D] tensors in ``w.kv_dtype``."""
    g = _gen(device, w.seed * 1_000_003 + 7919 * b + seed_offset)
    outs = []
    for _tensor in range(2):
        sigma = _sigma(w.Hkv, w.D, g, device)
        if w.gen == "walk":
            x = _walk(w.Hkv, T, w.D, sigma, w.step, w.jump_p, g, device)
        elif w.gen == "repeat":
            x = _windows(w.Hkv, T, w.D, sigma, w.step, g, device, p_walk=0.0, p_repeat=1.0)
        elif w.gen == "mixture":
            x = _windows(w.Hkv, T, w.D, sigma, w.step, g, device, p_walk=0.7, p_repeat=0.2)
        else:
            raise ValueError(w.gen)
        outs.append(x.to(w.kv_dtype))
    return outs[0], outs[1]


def gen_kv(w: Workload, device="cpu", T: int | None = None):
    """K, V as [B, Hkv, T, D] tensors in ``w.kv_dtype``."""
    T = w.T if T is None else T
    K = torch.empty((w.B, w.Hkv, T, w.D), dtype=w.kv_dtype, device=device)
    V = torch.empty_like(K)
    for b in range(w.B):
        K[b], V[b] = gen_kv_one(w, b, T, device)
    return K, V


def gen_q(w: Workload, device="cpu", step: int = 0) -> torch.Tensor:
    g = _gen(device, w.seed * 7 + 17 + step)
    return torch.randn((w.B, w.Hq, w.D), generator=g, device=device,
                       dtype=torch.float32).to(w.q_dtype)


def gen_lengths(w: Workload) -> list[int]:
    """Per-sequence context lengths (ragged workloads draw them uniformly)."""
    if w.ragged is None:
        return [w.T] * w.B
    g = _gen("cpu", w.seed + 99)
    lo, hi = w.ragged
    return [int(x) for x in torch.randint(lo, hi + 1, (w.B,), generator=g)]
