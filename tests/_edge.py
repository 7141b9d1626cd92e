"""Token sequences built to hit the corner cases of the Q4_0 block rule inside
the closed loop of Delta-KV (test infrastructure).

Page "영상 압축 기법을 KV 캐시에 적용해 Q4 양자화 오차를 10,000배 줄인
Delta-KV", section "핵심 아이디어": every kf-th token is an fp16 keyframe and
every other token stores the Q4_0 code of its difference from the
reconstructed previous token.  To make that difference equal a designed block
v, token p is x_p = x^_{p-1} + v, with x^_{p-1} taken from the oracle's own
incremental encoder.  The designed values are dyadic and each keyframe group
keeps one magnitude regime per 32-channel block, so the fp32 sum is exact and
the realised delta is v itself (the coverage count below checks what was
realised, not what was intended).

Designed blocks: the hand-worked golden blocks (tests/golden), rotated so
ties sit at low and at high lanes; +a/-a ties in both orders (the element at
-m clamps to code 15); exact half-way points (k + 1/2) d; all-zero deltas;
maxima whose scale m/-8 is an fp16 subnormal or rounds to zero; maxima whose
rounded subnormal scale is smaller than m/8 (codes below 0 clamp); large
blocks; plain random blocks.
"""
from __future__ import annotations

import json
from pathlib import Path

import numpy as np

D = 128
NB = 4
_GOLD = json.loads((Path(__file__).parent / "golden" / "quant_worked_examples.json").read_text())


def _golden_blocks():
    out = []
    for case in _GOLD["blocks"]:
        v = np.full(32, case.get("fill", 0.0), dtype=np.float64)
        for k, x in case["values_nonzero"].items():
            v[int(k)] = x
        out.append(v)
    return out


GOLDEN = _golden_blocks()

# regimes of one block within one keyframe group
R_DYADIC, R_TINY, R_RANDOM, R_LARGE = range(4)


def _pattern(rng, regime: int, k: int) -> np.ndarray:
    """The k-th designed delta block of a regime (float64, exact dyadic
    values except in the random regime)."""
    if regime == R_DYADIC:
        kind = k % 9
        s = 2.0 ** int(rng.integers(-2, 2))
        if kind < 4:                                 # golden blocks, rolled
            return np.roll(GOLDEN[kind], int(rng.choice([0, 7, 30, 31]))) * s
        if kind == 4:                                # +a / -a tie, lanes i < j
            v = rng.integers(-63, 64, 32) / 64.0 * s
            i, j = sorted(rng.choice(32, 2, replace=False))
            sg = rng.choice([-1.0, 1.0])
            v[i], v[j] = sg * s, -sg * s
            return v
        if kind == 5:                                # tie at the two highest lanes
            v = rng.integers(-63, 64, 32) / 64.0 * s
            sg = rng.choice([-1.0, 1.0])
            v[30], v[31] = sg * s, -sg * s
            return v
        if kind == 6:                                # exact halves (k + 1/2) d
            d = s / 8.0
            v = (rng.integers(-8, 8, 32) + 0.5) * d
            i = int(rng.integers(32))
            v[i] = rng.choice([-8.0, 8.0]) * d       # m = -/+ 8 d: d16 = +/- d exactly
            return v
        if kind == 7:                                # zero delta
            return np.zeros(32)
        v = rng.integers(-127, 128, 32) / 128.0 * s  # dyadic, general position
        return v
    if regime == R_TINY:
        kind = k % 5
        e = int(rng.integers(14, 26))                # m = c 2^-e: m/8 subnormal .. below 2^-25
        c = float(rng.choice([1.0, 1.25, 1.5, 1.75, 1.875]))
        m = c * 2.0 ** -e
        if kind == 4:
            return np.zeros(32)
        v = rng.integers(-64, 65, 32) / 64.0 * m
        i = int(rng.integers(32))
        v[i] = rng.choice([-1.0, 1.0]) * m
        if kind == 3:                                # tie with the opposite sign
            j = (i + 1 + int(rng.integers(31))) % 32
            v[j] = -v[i]
            if j < i:
                v[i], v[j] = v[j], v[i]
        return v
    if regime == R_LARGE:
        s = 2.0 ** int(rng.integers(6, 10))          # |x| up to ~2^10 (fp16 range)
        v = rng.integers(-255, 256, 32) / 256.0 * s
        if k % 2:
            i, j = sorted(rng.choice(32, 2, replace=False))
            v[i], v[j] = s, -s
        return v
    return rng.standard_normal(32) * 10.0 ** rng.uniform(-3, 0.5)


def edge_sequence(orc, T: int, kf: int, seed: int) -> np.ndarray:
    """[T, 128] fp32 tokens whose closed-loop deltas are the designed blocks."""
    rng = np.random.default_rng(seed)
    x = np.zeros((T, D), dtype=np.float32)
    seq = orc.DeltaSeq(T, D, kf)
    regime = np.zeros(NB, dtype=np.int64)
    count = 0
    for p in range(T):
        if p % kf == 0:
            regime = rng.integers(0, 4, NB)
            row = np.zeros(D, dtype=np.float64)
            for j in range(NB):                      # keyframe values exact in fp16
                if regime[j] == R_RANDOM:
                    row[32 * j:32 * j + 32] = rng.standard_normal(32)
                elif regime[j] == R_DYADIC:
                    row[32 * j:32 * j + 32] = rng.integers(-64, 65, 32) / 16.0
            row = row.astype(np.float16).astype(np.float64)
        else:
            prev = seq.xhat[p - 1].astype(np.float64)
            pat = np.concatenate([_pattern(rng, int(regime[j]), count + 3 * j) for j in range(NB)])
            row = prev + pat
            count += 1
        x[p] = row.astype(np.float32)
        seq.append(x[p:p + 1])
    return x


def constant_sequence(T: int, seed: int) -> np.ndarray:
    """[T, 128] a constant fp16-representable token: every delta is zero."""
    rng = np.random.default_rng(seed)
    row = (rng.standard_normal(D) * 2.0).astype(np.float16).astype(np.float32)
    return np.repeat(row[None], T, axis=0)


def coverage(x: np.ndarray, kf: int, enc) -> dict:
    """Counts of the corner cases the oracle's encoding `enc` (a DeltaSeq of x)
    actually met: the realised delta of every delta block is recomputed from
    x and the oracle's reconstruction with numpy fp32 arithmetic."""
    T = x.shape[0]
    c = dict(tie=0, tie_high=0, zero_block=0, half=0, clamp15=0, clamp0=0, sub_d=0,
             zero_d_nonzero=0, delta_rows=0)
    for p in range(1, T):
        if p % kf == 0:
            continue
        c["delta_rows"] += 1
        delta = (x[p] - enc.xhat[p - 1]).astype(np.float32)
        for j in range(NB):
            v = delta[32 * j:32 * j + 32]
            bits = int(enc.scales[p, j])
            codes = enc.codes[p, 32 * j:32 * j + 32].astype(np.int64)
            a = np.abs(v)
            mx = a.max()
            at = np.flatnonzero(a == mx)
            if mx > 0 and len(at) > 1 and (np.sign(v[at]) != np.sign(v[at[0]])).any():
                c["tie"] += 1
                if at.max() >= 30:
                    c["tie_high"] += 1
            if mx == 0:
                c["zero_block"] += 1
                continue
            d = np.float32(np.uint16(bits).view(np.float16))
            if d == 0:
                c["zero_d_nonzero"] += 1
                continue
            if (bits & 0x7C00) == 0:
                c["sub_d"] += 1
            q = (v / d).astype(np.float32)
            if (q - np.floor(q) == 0.5).any():
                c["half"] += 1
            u = (q + np.float32(8.5)).astype(np.float32)
            if ((codes == 15) & (u >= 16)).any():
                c["clamp15"] += 1
            if ((codes == 0) & (u < 0)).any():
                c["clamp0"] += 1
    return c
