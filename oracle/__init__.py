"""CPU oracle for the Delta-KV decode path -- TEST INFRASTRUCTURE ONLY.

This package wraps ``dkv_oracle.c`` (plain C: IEEE binary32 quantiser steps in
source order, binary64 attention) through ctypes.  It is the independent
statement of the method that the CUDA library is checked against.  Only the
test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import it; the library never does.

Every function here restates one step of the method as the web pages describe
it (see the C source header for the citations):

* ``quant_block``      -- the Q4_0 block rule on 32 values;
* ``delta_encode``     -- keyframe every kf-th token (fp16), closed-loop 4-bit
                          deltas against the reconstructed previous token;
* ``delta_append``     -- the same loop continued from a saved state;
* ``delta_decode``     -- reconstruction from the stored codes alone;
* ``q4_encode`` / ``f16_encode`` -- the two comparator caches;
* ``attn``             -- one decode step of softmax attention, binary64;
* ``lr_encode``        -- long-range reference encoding: fp16 references at a
                          fixed stride, each other token the Q4_0 residual
                          against the mean of its most similar references
                          (the training-free part of DeltaKV).

Every function is pinned by tests under ``tests/test_oracle_*.py`` against
closed forms, invariants, brute force and library routines (numpy float16
conversion, numpy float64 softmax).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "dkv_oracle.c"
_LIB_PATH = _HERE / "_build" / "liboracle.so"
BLOCK = 32

_lib = None


def build(force: bool = False) -> Path:
    """Compile the C oracle with gcc (no fast-math, no FMA contraction)."""
    _LIB_PATH.parent.mkdir(parents=True, exist_ok=True)
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".{os.getpid()}.tmp.so")
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-fno-finite-math-only", str(_SRC), "-lm", "-o", str(tmp)]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB_PATH))
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.or_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.or_f16_to_f32.restype = ctypes.c_float
        lib.or_f32_to_f16.argtypes = [ctypes.c_float]
        lib.or_f32_to_f16.restype = ctypes.c_uint16
        lib.or_quant_block.argtypes = [P, P, P]
        lib.or_delta_encode_range.argtypes = [i, i, i, i, P, P, P, P, P, P]
        lib.or_delta_decode.argtypes = [i, i, i, P, P, P, P]
        lib.or_q4_encode.argtypes = [i, i, P, P, P, P]
        lib.or_f16_encode.argtypes = [i, i, P, P, P]
        lib.or_attn.argtypes = [i, i, i, P, P, P, ctypes.c_double, P]
        lib.or_lr_encode.argtypes = [i, i, i, i, P, P, P, P, P, P]
        for f in ("or_quant_block", "or_delta_encode_range", "or_delta_decode",
                  "or_q4_encode", "or_f16_encode", "or_attn", "or_lr_encode"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# binary16 helpers
# --------------------------------------------------------------------------
def f32_to_f16_bits(x) -> np.ndarray:
    """Round each binary32 value to binary16 (nearest, ties to even); bits."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    flat_in, flat_out = x.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = lib.or_f32_to_f16(float(flat_in[i]))
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    lib = _load()
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    fi, fo = h.reshape(-1), out.reshape(-1)
    for i in range(fi.size):
        fo[i] = lib.or_f16_to_f32(int(fi[i]))
    return out


# --------------------------------------------------------------------------
# quantiser
# --------------------------------------------------------------------------
def quant_block(v) -> tuple[int, np.ndarray]:
    """Q4_0 rule on one block of 32 values -> (scale bits d16, codes[32])."""
    lib = _load()
    v = np.ascontiguousarray(v, dtype=np.float32)
    assert v.shape == (BLOCK,)
    d16 = np.zeros(1, dtype=np.uint16)
    codes = np.zeros(BLOCK, dtype=np.uint8)
    lib.or_quant_block(_p(v), _p(d16), _p(codes))
    return int(d16[0]), codes


# --------------------------------------------------------------------------
# Delta-KV encoder / decoder for one sequence of one tensor
# --------------------------------------------------------------------------
class DeltaSeq:
    """Oracle cache of one (batch, kv-head, tensor) sequence.

    Arrays are indexed by absolute position up to ``cap``:
    ``kfr[g, D]`` (fp16 bits of keyframe g), ``scales[p, D/32]`` (fp16 bits),
    ``codes[p, D]`` (0..15), ``xhat[p, D]`` (binary32 reconstruction) and
    ``state[D]`` (reconstruction of the last encoded position).  Keyframe
    rows of ``scales``/``codes`` stay zero.
    """

    def __init__(self, cap: int, D: int, kf: int):
        assert D % BLOCK == 0 and kf >= 1
        self.cap, self.D, self.kf = cap, D, kf
        ng = (cap + kf - 1) // kf
        self.kfr = np.zeros((ng, D), dtype=np.uint16)
        self.scales = np.zeros((cap, D // BLOCK), dtype=np.uint16)
        self.codes = np.zeros((cap, D), dtype=np.uint8)
        self.xhat = np.zeros((cap, D), dtype=np.float32)
        self.state = np.zeros(D, dtype=np.float32)
        self.length = 0

    def append(self, x) -> None:
        lib = _load()
        x = np.ascontiguousarray(x, dtype=np.float32)
        n = x.shape[0]
        assert x.shape == (n, self.D) and self.length + n <= self.cap
        lib.or_delta_encode_range(self.length, n, self.D, self.kf, _p(x), _p(self.kfr),
                                  _p(self.scales), _p(self.codes), _p(self.xhat),
                                  _p(self.state))
        self.length += n


def delta_encode(x, kf: int, cap: int | None = None) -> DeltaSeq:
    x = np.asarray(x, dtype=np.float32)
    T, D = x.shape
    s = DeltaSeq(cap if cap is not None else T, D, kf)
    s.append(x)
    return s


def delta_decode(T: int, kf: int, kfr, scales, codes) -> np.ndarray:
    """Reconstruct positions [0, T) from stored keyframes, scales and codes."""
    lib = _load()
    kfr = np.ascontiguousarray(kfr, dtype=np.uint16)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    D = codes.shape[1]
    out = np.zeros((T, D), dtype=np.float32)
    lib.or_delta_decode(T, D, kf, _p(kfr), _p(scales), _p(codes), _p(out))
    return out


def q4_encode(x):
    """Plain Q4_0 comparator -> (scales[T, D/32] bits, codes[T, D], xhat[T, D])."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    T, D = x.shape
    scales = np.zeros((T, D // BLOCK), dtype=np.uint16)
    codes = np.zeros((T, D), dtype=np.uint8)
    xhat = np.zeros((T, D), dtype=np.float32)
    lib.or_q4_encode(T, D, _p(x), _p(scales), _p(codes), _p(xhat))
    return scales, codes, xhat


def f16_encode(x):
    """F16 comparator -> (bits[T, D], xhat[T, D])."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    T, D = x.shape
    bits = np.zeros((T, D), dtype=np.uint16)
    xhat = np.zeros((T, D), dtype=np.float32)
    lib.or_f16_encode(T, D, _p(x), _p(bits), _p(xhat))
    return bits, xhat


def lr_encode(x, s: int, m: int) -> dict:
    """Long-range reference encoding of one [T, D] sequence (stride s, the m
    most similar references; see ``or_lr_encode`` in the C source) ->
    dict(ref[T, m] int32, kfr[ceil(T/s), D] fp16 bits, scales[T, D/32] fp16
    bits, codes[T, D], xhat[T, D] binary32)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    T, D = x.shape
    assert D % BLOCK == 0 and s >= 1 and m >= 1
    ng = max(1, (T + s - 1) // s)
    out = {"ref": np.zeros((T, m), np.int32), "kfr": np.zeros((ng, D), np.uint16),
           "scales": np.zeros((T, D // BLOCK), np.uint16), "codes": np.zeros((T, D), np.uint8),
           "xhat": np.zeros((T, D), np.float32)}
    lib.or_lr_encode(T, D, s, m, _p(x), _p(out["ref"]), _p(out["kfr"]), _p(out["scales"]),
                     _p(out["codes"]), _p(out["xhat"]))
    return out


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def attn(q, khat, vhat, scale: float) -> np.ndarray:
    """One decode step for the G query heads of one KV head, binary64.

    q [G, D] (any float dtype, used exactly), khat/vhat [T, D] binary32.
    Returns o [G, D] float64.
    """
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    khat = np.ascontiguousarray(khat, dtype=np.float32)
    vhat = np.ascontiguousarray(vhat, dtype=np.float32)
    G, D = q.shape
    T = khat.shape[0]
    assert khat.shape == (T, D) and vhat.shape == (T, D)
    out = np.zeros((G, D), dtype=np.float64)
    lib.or_attn(T, D, G, _p(q), _p(khat), _p(vhat), float(scale), _p(out))
    return out


# --------------------------------------------------------------------------
# whole-cache helpers used by the parity tests and the CPU baseline
# --------------------------------------------------------------------------
def encode_cache(fmt: str, x, kf: int = 32, n_refs: int = 1):
    """Encode one [T, D] tensor in format ``fmt`` ('delta', 'q4', 'fp16', or
    'lr': long-range references at stride kf, the n_refs nearest).

    Returns a dict with the reconstruction ``xhat`` and the stored fields.
    """
    x = np.asarray(x, dtype=np.float32)
    if fmt == "lr":
        return lr_encode(x, kf, n_refs)
    if fmt == "delta":
        s = delta_encode(x, kf)
        return {"xhat": s.xhat, "kfr": s.kfr, "scales": s.scales, "codes": s.codes,
                "state": s.state}
    if fmt == "q4":
        scales, codes, xhat = q4_encode(x)
        return {"xhat": xhat, "scales": scales, "codes": codes}
    if fmt == "fp16":
        bits, xhat = f16_encode(x)
        return {"xhat": xhat, "bits": bits}
    raise ValueError(fmt)


def decode_attention(fmt: str, q, K, V, kf: int, scale: float, lengths=None):
    """Full oracle of one decode step over a batch.

    q [B, Hq, D], K/V [B, Hkv, T, D] (already-exact float values), ``lengths``
    per batch entry (default T).  Returns o [B, Hq, D] float64.
    """
    q = np.asarray(q)
    B, Hq, D = q.shape
    Hkv, T = K.shape[1], K.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        L = T if lengths is None else int(lengths[b])
        for h in range(Hkv):
            kh = encode_cache(fmt, K[b, h, :L], kf)["xhat"]
            vh = encode_cache(fmt, V[b, h, :L], kf)["xhat"]
            out[b, h * G:(h + 1) * G] = attn(q[b, h * G:(h + 1) * G], kh, vh, scale)
    return out
