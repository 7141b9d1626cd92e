"""Python binding of the Delta-KV decode library (``include/dkv.h``).

Argument marshalling only: every step of the encode, append and decode path
runs in the library's CUDA kernels (``_lib/libdkv.so``, built for sm_100a).
PyTorch is used for device memory and streams.  If the shared library is
missing, every call raises -- there is no CPU fallback.

The functions carry the C names (``dkv_encode`` ...) and take either raw
integers (device pointers, a stream handle) or torch tensors / streams.
``Cache`` is a small convenience that allocates a cache with torch and keeps
its ``dkv_cache`` descriptor.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "_lib" / "libdkv.so"
# the bounds-checked build (DKV_CHECKED=1, for tests): selected by setting
# DKV_LIBRARY=checked in the environment before the first load()
CHECKED_LIB_PATH = _PKG / "_lib" / "libdkv_checked.so"

DKV_OK, DKV_EINVAL, DKV_EALIGN, DKV_ECAPACITY, DKV_EUNSUPPORTED, DKV_ECUDA, DKV_EDEVICE = range(7)
DKV_FMT_FP16, DKV_FMT_Q4_0, DKV_FMT_DELTA = 0, 1, 2
DKV_F32, DKV_F16, DKV_BF16 = 0, 1, 2
DEV_BAD_SEQLEN, DEV_CAPACITY, DEV_TIMEOUT, DEV_BAD_HEADS, DEV_BAD_PAGE = 0x1, 0x2, 0x4, 0x8, 0x10
DEV_BOUNDS = 0x20
FORMATS = {"fp16": DKV_FMT_FP16, "q4": DKV_FMT_Q4_0, "delta": DKV_FMT_DELTA}


class DkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


class dkv_cache_desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("kf", ctypes.c_int32),
                ("max_ctx", ctypes.c_int32), ("fmt", ctypes.c_int32)]


class dkv_lr_tensor(ctypes.Structure):
    _fields_ = [("ref", ctypes.c_void_p), ("ref_values", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("codes", ctypes.c_void_p)]


class dkv_cache(ctypes.Structure):
    _fields_ = [("desc", dkv_cache_desc), ("base", ctypes.c_void_p), ("bytes", ctypes.c_size_t),
                ("seq_stride", ctypes.c_size_t), ("rec_bytes", ctypes.c_size_t),
                ("n_groups", ctypes.c_int32), ("reserved0", ctypes.c_int32),
                ("off_data", ctypes.c_size_t), ("off_state", ctypes.c_size_t),
                ("off_seqlen", ctypes.c_size_t), ("off_header", ctypes.c_size_t),
                ("pool", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("page_bytes", ctypes.c_size_t), ("n_pages", ctypes.c_int64),
                ("page_groups", ctypes.c_int32), ("max_pages", ctypes.c_int32)]


_lib = None
EXPORTS = ["dkv_abi_version", "dkv_cache_bytes", "dkv_cache_init", "dkv_encode", "dkv_append",
           "dkv_decode_workspace_bytes", "dkv_decode_attn", "dkv_decode_attn_split",
           "dkv_decode_attn_merge", "dkv_export_canonical", "dkv_dequantize",
           "dkv_get_device_status", "dkv_status_str", "dkv_decode_attn_noalloc",
           "dkv_debug_set_fault", "dkv_cache_meta_bytes", "dkv_page_bytes",
           "dkv_cache_init_paged", "dkv_decode_workspace_bytes_mq", "dkv_decode_attn_mq",
           "dkv_append_decode_attn", "dkv_append_decode_attn_split",
           "dkv_append_decode_attn_merge", "dkv_lr_encode", "dkv_lr_decode_workspace_bytes",
           "dkv_lr_decode_attn", "dkv_debug_division_check"]


def load():
    """Load ``libdkv.so`` (raises if it has not been built), or the
    bounds-checked ``libdkv_checked.so`` when DKV_LIBRARY=checked."""
    global _lib
    if _lib is not None:
        return _lib
    import os
    path = CHECKED_LIB_PATH if os.environ.get("DKV_LIBRARY") == "checked" else LIB_PATH
    if not path.exists():
        raise RuntimeError(f"{path.name} not built ({path}); run __graft_entry__.build() "
                           "or python -m delta_quantized_kv_b200.build")
    lib = ctypes.CDLL(str(path))
    P, S, I, F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_float
    PC = ctypes.POINTER(dkv_cache)
    PD = ctypes.POINTER(dkv_cache_desc)
    sig = {
        "dkv_abi_version": ([], I),
        "dkv_cache_bytes": ([PD], S),
        "dkv_cache_init": ([PD, P, S, PC, P], I),
        "dkv_encode": ([PC, P, P, I, P, I, P], I),
        "dkv_append": ([PC, P, P, I, I, P], I),
        "dkv_decode_workspace_bytes": ([PD, I], S),
        "dkv_decode_attn": ([PC, P, I, I, F, P, P, S, P], I),
        "dkv_decode_attn_split": ([PC, P, I, I, F, P, S, P], I),
        "dkv_decode_attn_merge": ([PC, I, P, P, S, P], I),
        "dkv_export_canonical": ([PC, P, P, P, P, P], I),
        "dkv_dequantize": ([PC, P, P], I),
        "dkv_get_device_status": ([PC, ctypes.POINTER(I), P], I),
        "dkv_status_str": ([I], ctypes.c_char_p),
        "dkv_decode_attn_noalloc": ([PC, P, I, I, F, P, P], I),
        "dkv_debug_set_fault": ([I], None),
        "dkv_cache_meta_bytes": ([PD], S),
        "dkv_page_bytes": ([PD, I], S),
        "dkv_cache_init_paged": ([PD, I, P, ctypes.c_int64, P, I, P, S, PC, P], I),
        "dkv_decode_workspace_bytes_mq": ([PD, I, I], S),
        "dkv_decode_attn_mq": ([PC, P, I, I, I, F, P, P, S, P], I),
        "dkv_append_decode_attn": ([PC, P, P, I, I, P, I, I, F, P, P, S, P], I),
        "dkv_append_decode_attn_split": ([PC, P, P, I, I, P, I, I, F, P, S, P], I),
        "dkv_append_decode_attn_merge": ([PC, I, I, P, P, S, P], I),
        "dkv_lr_encode": ([P, I, I, I, I, I, P, P, P, P, P, P], I),
        "dkv_lr_decode_workspace_bytes": ([I, I, I, I], S),
        "dkv_debug_division_check": ([P, I, P, P], I),
        "dkv_lr_decode_attn": ([ctypes.POINTER(dkv_lr_tensor), ctypes.POINTER(dkv_lr_tensor),
                                I, I, I, I, I, P, P, I, I, F, P, P, S, P], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def status_str(s: int) -> str:
    return load().dkv_status_str(int(s)).decode()


def _ptr(x):
    """Device pointer of a tensor (or an int / None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: DKV_F32, torch.float16: DKV_F16, torch.bfloat16: DKV_BF16}[t]


def _check(s: int, what: str):
    if s != DKV_OK:
        raise DkvError(s, what)


# ---------------------------------------------------------------------------
# the C functions, same names
# ---------------------------------------------------------------------------
def dkv_abi_version() -> int:
    return load().dkv_abi_version()


def dkv_cache_bytes(desc: dkv_cache_desc) -> int:
    return load().dkv_cache_bytes(ctypes.byref(desc))


def dkv_cache_init(desc: dkv_cache_desc, dev, nbytes: int, stream=None) -> dkv_cache:
    out = dkv_cache()
    _check(load().dkv_cache_init(ctypes.byref(desc), _ptr(dev), nbytes, ctypes.byref(out),
                                 _stream(stream)), "dkv_cache_init")
    return out


def dkv_cache_meta_bytes(desc: dkv_cache_desc) -> int:
    return load().dkv_cache_meta_bytes(ctypes.byref(desc))


def dkv_page_bytes(desc: dkv_cache_desc, page_groups: int) -> int:
    return load().dkv_page_bytes(ctypes.byref(desc), page_groups)


def dkv_cache_init_paged(desc: dkv_cache_desc, page_groups: int, pool, n_pages: int,
                         block_table, max_pages: int, meta, meta_bytes: int,
                         stream=None) -> dkv_cache:
    out = dkv_cache()
    _check(load().dkv_cache_init_paged(ctypes.byref(desc), page_groups, _ptr(pool), n_pages,
                                       _ptr(block_table), max_pages, _ptr(meta), meta_bytes,
                                       ctypes.byref(out), _stream(stream)),
           "dkv_cache_init_paged")
    return out


def dkv_encode(cache: dkv_cache, K, V, dtype=None, seq_lens=None, T=None, stream=None) -> None:
    dtype = _dtype_code(K.dtype) if dtype is None else dtype
    T = K.shape[2] if T is None else T
    _check(load().dkv_encode(ctypes.byref(cache), _ptr(K), _ptr(V), dtype, _ptr(seq_lens), T,
                             _stream(stream)), "dkv_encode")


def dkv_append(cache: dkv_cache, K_new, V_new, dtype=None, n_new=None, stream=None) -> None:
    dtype = _dtype_code(K_new.dtype) if dtype is None else dtype
    n_new = K_new.shape[2] if n_new is None else n_new
    _check(load().dkv_append(ctypes.byref(cache), _ptr(K_new), _ptr(V_new), dtype, n_new,
                             _stream(stream)), "dkv_append")


def dkv_decode_workspace_bytes(desc: dkv_cache_desc, n_q_heads: int) -> int:
    return load().dkv_decode_workspace_bytes(ctypes.byref(desc), n_q_heads)


def dkv_decode_attn(cache: dkv_cache, Q, q_dtype, n_q_heads, softmax_scale, out, workspace,
                    ws_bytes, stream=None) -> None:
    _check(load().dkv_decode_attn(ctypes.byref(cache), _ptr(Q), q_dtype, n_q_heads,
                                  softmax_scale, _ptr(out), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "dkv_decode_attn")


def dkv_decode_workspace_bytes_mq(desc: dkv_cache_desc, n_q_heads: int, n_queries: int) -> int:
    return load().dkv_decode_workspace_bytes_mq(ctypes.byref(desc), n_q_heads, n_queries)


def dkv_decode_attn_mq(cache: dkv_cache, Q, q_dtype, n_q_heads, n_queries, softmax_scale, out,
                       workspace, ws_bytes, stream=None) -> None:
    _check(load().dkv_decode_attn_mq(ctypes.byref(cache), _ptr(Q), q_dtype, n_q_heads, n_queries,
                                     softmax_scale, _ptr(out), _ptr(workspace), ws_bytes,
                                     _stream(stream)), "dkv_decode_attn_mq")


def dkv_append_decode_attn(cache: dkv_cache, K_new, V_new, kv_dtype, n_new, Q, q_dtype,
                           n_q_heads, softmax_scale, out, workspace, ws_bytes,
                           stream=None) -> None:
    _check(load().dkv_append_decode_attn(ctypes.byref(cache), _ptr(K_new), _ptr(V_new), kv_dtype,
                                         n_new, _ptr(Q), q_dtype, n_q_heads, softmax_scale,
                                         _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)),
           "dkv_append_decode_attn")


def dkv_append_decode_attn_split(cache: dkv_cache, K_new, V_new, kv_dtype, n_new, Q, q_dtype,
                                 n_q_heads, softmax_scale, workspace, ws_bytes,
                                 stream=None) -> None:
    _check(load().dkv_append_decode_attn_split(ctypes.byref(cache), _ptr(K_new), _ptr(V_new),
                                               kv_dtype, n_new, _ptr(Q), q_dtype, n_q_heads,
                                               softmax_scale, _ptr(workspace), ws_bytes,
                                               _stream(stream)), "dkv_append_decode_attn_split")


def dkv_append_decode_attn_merge(cache: dkv_cache, n_new, n_q_heads, out, workspace, ws_bytes,
                                 stream=None) -> None:
    _check(load().dkv_append_decode_attn_merge(ctypes.byref(cache), n_new, n_q_heads, _ptr(out),
                                               _ptr(workspace), ws_bytes, _stream(stream)),
           "dkv_append_decode_attn_merge")


def lr_encode(X, stride: int, n_refs: int, stream=None) -> dict:
    """Long-range reference encoding (dkv_lr_encode) of X [n_seq, T, 128] on
    the GPU -> dict of device tensors ref, ref_values, scales, codes, xhat in
    the canonical layouts."""
    import torch
    if X.dim() != 3 or X.shape[2] != 128:
        raise ValueError("lr_encode takes X of shape [n_seq, T, 128]")
    n_seq, T, Dh = X.shape
    if stride < 1 or not 1 <= n_refs <= 8:
        raise DkvError(DKV_EINVAL, "dkv_lr_encode")
    ng = -(-T // stride)
    dev = X.device
    out = {"ref": torch.empty((n_seq, T, n_refs), dtype=torch.int32, device=dev),
           "ref_values": torch.empty((n_seq, ng, Dh), dtype=torch.int16, device=dev),
           "scales": torch.empty((n_seq, T, Dh // 32), dtype=torch.int16, device=dev),
           "codes": torch.empty((n_seq, T, Dh), dtype=torch.uint8, device=dev),
           "xhat": torch.empty((n_seq, T, Dh), dtype=torch.float32, device=dev)}
    X = X.contiguous()
    _check(load().dkv_lr_encode(_ptr(X), _dtype_code(X.dtype), n_seq, T, stride, n_refs,
                                _ptr(out["ref"]), _ptr(out["ref_values"]), _ptr(out["scales"]),
                                _ptr(out["codes"]), _ptr(out["xhat"]), _stream(stream)),
           "dkv_lr_encode")
    return out


def dkv_lr_decode_workspace_bytes(batch: int, n_kv_heads: int, T: int, stride: int) -> int:
    return load().dkv_lr_decode_workspace_bytes(batch, n_kv_heads, T, stride)


def _lr_view(enc) -> dkv_lr_tensor:
    return dkv_lr_tensor(_ptr(enc["ref"]), _ptr(enc["ref_values"]), _ptr(enc["scales"]),
                         _ptr(enc["codes"]))


def lr_decode_attn(enc_k: dict, enc_v: dict, Q, softmax_scale: float, stride: int,
                   n_kv_heads: int, lens=None, out=None, workspace=None, stream=None):
    """Decode attention over long-range reference encodings (dkv_lr_decode_attn).
    enc_k, enc_v: the dicts `lr_encode` returns for K and V, each encoding
    [B * n_kv_heads, T, 128] sequences (sequence = batch entry * n_kv_heads +
    kv head) with the same stride and n_refs; Q [B, n_q_heads, 128];
    lens: device int32 [B] or None.  Returns fp32 [B, n_q_heads, 128]."""
    import torch
    n_seq, T, n_refs = enc_k["ref"].shape
    B = n_seq // n_kv_heads
    Hq = Q.shape[1]
    if out is None:
        out = torch.empty((B, Hq, 128), dtype=torch.float32, device=Q.device)
    nb = dkv_lr_decode_workspace_bytes(B, n_kv_heads, T, stride)
    if workspace is None:
        workspace = torch.empty(nb // 4 + 64, dtype=torch.float32, device=Q.device)
    kv, vv = _lr_view(enc_k), _lr_view(enc_v)
    Q = Q.contiguous()
    _check(load().dkv_lr_decode_attn(ctypes.byref(kv), ctypes.byref(vv), B, n_kv_heads, T, stride,
                                     n_refs, _ptr(lens), _ptr(Q), _dtype_code(Q.dtype), Hq,
                                     softmax_scale, _ptr(out), _ptr(workspace),
                                     workspace.numel() * 4, _stream(stream)),
           "dkv_lr_decode_attn")
    return out


def dkv_decode_attn_split(cache: dkv_cache, Q, q_dtype, n_q_heads, softmax_scale, workspace,
                          ws_bytes, stream=None) -> None:
    _check(load().dkv_decode_attn_split(ctypes.byref(cache), _ptr(Q), q_dtype, n_q_heads,
                                        softmax_scale, _ptr(workspace), ws_bytes,
                                        _stream(stream)), "dkv_decode_attn_split")


def dkv_decode_attn_merge(cache: dkv_cache, n_q_heads, out, workspace, ws_bytes,
                          stream=None) -> None:
    _check(load().dkv_decode_attn_merge(ctypes.byref(cache), n_q_heads, _ptr(out),
                                        _ptr(workspace), ws_bytes, _stream(stream)),
           "dkv_decode_attn_merge")


def dkv_decode_attn_noalloc(cache: dkv_cache, Q, q_dtype, n_q_heads, softmax_scale, out,
                            stream=None) -> None:
    """Decode step that needs no workspace: the partial records go to a fixed
    16 MiB array the library keeps on each GPU (for callers that cannot
    allocate device memory when they decode, e.g. under graph capture).
    Calls overlapping on the GPU race on that array."""
    _check(load().dkv_decode_attn_noalloc(ctypes.byref(cache), _ptr(Q), q_dtype, n_q_heads,
                                          softmax_scale, _ptr(out), _stream(stream)),
           "dkv_decode_attn_noalloc")


def dkv_export_canonical(cache: dkv_cache, codes=None, scales=None, keyframes=None, state=None,
                         stream=None) -> None:
    _check(load().dkv_export_canonical(ctypes.byref(cache), _ptr(codes), _ptr(scales),
                                       _ptr(keyframes), _ptr(state), _stream(stream)),
           "dkv_export_canonical")


def dkv_dequantize(cache: dkv_cache, out, stream=None) -> None:
    _check(load().dkv_dequantize(ctypes.byref(cache), _ptr(out), _stream(stream)),
           "dkv_dequantize")


def dkv_debug_set_fault(mode: int) -> None:
    """Test support: mode 1 makes later split launches time out by design."""
    load().dkv_debug_set_fault(int(mode))


def dkv_debug_division_check(u, mismatches, stream=None) -> None:
    """Test support: count (into the device uint64 `mismatches`) the encoder
    quotients that differ from IEEE division, over every fp16 divisor and the
    dividends RN(u_i b) and their neighbours (u: device fp32)."""
    _check(load().dkv_debug_division_check(_ptr(u), u.numel(), _ptr(mismatches),
                                           _stream(stream)), "dkv_debug_division_check")


def dkv_get_device_status(cache: dkv_cache, stream=None) -> int:
    word = ctypes.c_int32(0)
    s = load().dkv_get_device_status(ctypes.byref(cache), ctypes.byref(word), _stream(stream))
    if s not in (DKV_OK, DKV_EDEVICE):
        raise DkvError(s, "dkv_get_device_status")
    return word.value


# ---------------------------------------------------------------------------
# convenience wrapper (torch allocations)
# ---------------------------------------------------------------------------
class Cache:
    """A Delta-KV (or comparator) cache in torch-allocated device memory."""

    def __init__(self, batch, n_kv_heads, max_ctx, fmt="delta", kf=32, head_dim=128,
                 device="cuda", stream=None, page_groups=None, n_pages=None,
                 block_table=None, page_seed=0):
        """page_groups: a paged cache (delta format) with pages of page_groups
        keyframe groups; the pool holds n_pages pages (default: exactly the
        pages every sequence needs at max_ctx) and block_table ([batch,
        max_pages] int32, default: a seeded random assignment of distinct
        pages) maps each sequence's groups to pages."""
        import torch
        self.desc = dkv_cache_desc(batch, n_kv_heads, head_dim, kf, max_ctx,
                                   FORMATS[fmt] if isinstance(fmt, str) else fmt)
        if page_groups:
            mb = dkv_cache_meta_bytes(self.desc)
            pb = dkv_page_bytes(self.desc, page_groups)
            if mb == 0 or pb == 0:
                raise DkvError(DKV_EINVAL, "dkv_cache_meta_bytes / dkv_page_bytes")
            n_groups = -(-max_ctx // kf)
            max_pages = -(-n_groups // page_groups)
            if n_pages is None:
                n_pages = batch * max_pages
            if block_table is None:
                g = torch.Generator().manual_seed(page_seed)
                perm = torch.randperm(n_pages, generator=g)[:batch * max_pages]
                block_table = perm.view(batch, max_pages).to(torch.int32)
            self.block_table = block_table.to(device=device, dtype=torch.int32).contiguous()
            self.buf = torch.empty(mb + 256, dtype=torch.uint8, device=device)
            self.pool = torch.empty(n_pages * pb + 256, dtype=torch.uint8, device=device)
            base = (self.buf.data_ptr() + 255) // 256 * 256
            pool = (self.pool.data_ptr() + 255) // 256 * 256
            self.c = dkv_cache_init_paged(self.desc, page_groups, pool, n_pages,
                                          self.block_table, max_pages, base, mb, stream)
        else:
            nbytes = dkv_cache_bytes(self.desc)
            if nbytes == 0:
                raise DkvError(DKV_EINVAL, "dkv_cache_bytes")
            self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
            base = (self.buf.data_ptr() + 255) // 256 * 256
            self.c = dkv_cache_init(self.desc, base, nbytes, stream)
        self._ws = None
        self._ws_heads = None
        self.device = device

    @property
    def fmt(self):
        return self.desc.fmt

    def encode(self, K, V, seq_lens=None, stream=None):
        dkv_encode(self.c, K, V, seq_lens=seq_lens, stream=stream)

    def append(self, K_new, V_new, stream=None):
        dkv_append(self.c, K_new, V_new, stream=stream)

    def workspace(self, n_q_heads):
        import torch
        if self._ws is None or self._ws_heads != n_q_heads:
            nb = dkv_decode_workspace_bytes(self.desc, n_q_heads)
            if nb == 0:
                raise DkvError(DKV_ECUDA, "dkv_decode_workspace_bytes")
            self._ws = torch.zeros(nb // 4 + 64, dtype=torch.float32, device=self.device)
            self._ws_heads = n_q_heads
        return self._ws

    def decode_attn(self, Q, softmax_scale, out=None, stream=None):
        import torch
        B, Hq, Dh = Q.shape
        if out is None:
            out = torch.empty((B, Hq, Dh), dtype=torch.float32, device=Q.device)
        ws = self.workspace(Hq)
        dkv_decode_attn(self.c, Q, _dtype_code(Q.dtype), Hq, softmax_scale, out, ws,
                        ws.numel() * 4, stream)
        return out

    def workspace_mq(self, n_q_heads, n_queries):
        import torch
        key = ("mq", n_q_heads, n_queries)
        ws = getattr(self, "_ws_mq", {}).get(key)
        if ws is None:
            nb = dkv_decode_workspace_bytes_mq(self.desc, n_q_heads, n_queries)
            if nb == 0:
                raise DkvError(DKV_EINVAL, "dkv_decode_workspace_bytes_mq")
            ws = torch.zeros(nb // 4 + 64, dtype=torch.float32, device=self.device)
            self._ws_mq = {key: ws}
        return ws

    def decode_attn_mq(self, Q, softmax_scale, out=None, stream=None):
        """Q: [B, n_queries, Hq, D]; query t attends causally (see
        dkv_decode_attn_mq).  Returns fp32 [B, n_queries, Hq, D]."""
        import torch
        B, nq, Hq, Dh = Q.shape
        if out is None:
            out = torch.empty((B, nq, Hq, Dh), dtype=torch.float32, device=Q.device)
        ws = self.workspace_mq(Hq, nq)
        dkv_decode_attn_mq(self.c, Q.contiguous(), _dtype_code(Q.dtype), Hq, nq, softmax_scale,
                           out, ws, ws.numel() * 4, stream)
        return out

    def append_decode_attn(self, K_new, V_new, Q, softmax_scale, out=None, stream=None):
        """Fused append + decode (dkv_append_decode_attn): K_new, V_new
        [B, Hkv, n_new, D]; Q [B, Hq, D] (n_new = 1) or [B, n_new, Hq, D].
        Returns fp32 of Q's shape."""
        import torch
        n_new = K_new.shape[2]
        Hq = Q.shape[-2]
        if Q.dim() == 3 and n_new != 1:
            raise ValueError("Q of shape [B, Hq, D] takes one new token per sequence")
        if Q.dim() == 4 and Q.shape[1] != n_new:
            raise ValueError("Q must hold one query per new token")
        if out is None:
            out = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
        ws = self.workspace_mq(Hq, n_new)
        dkv_append_decode_attn(self.c, K_new, V_new, _dtype_code(K_new.dtype), n_new,
                               Q.contiguous(), _dtype_code(Q.dtype), Hq, softmax_scale, out, ws,
                               ws.numel() * 4, stream)
        return out

    def seq_lens(self):
        import torch
        n = self.desc.batch
        base = self.c.base + self.c.off_seqlen
        off = base - self.buf.data_ptr()
        return self.buf[off:off + 4 * n].view(torch.int32).clone()

    def export(self, stream=None):
        """Canonical fields as torch tensors (codes, scales, keyframes, state)."""
        import torch
        d = self.desc
        B, H, cap = d.batch, d.n_kv_heads, d.max_ctx
        dev = self.device
        out = {}
        if d.fmt in (DKV_FMT_DELTA, DKV_FMT_Q4_0):
            out["codes"] = torch.zeros((B, H, 2, cap, 128), dtype=torch.uint8, device=dev)
            out["scales"] = torch.zeros((B, H, 2, cap, 4), dtype=torch.int16, device=dev)
        if d.fmt == DKV_FMT_DELTA:
            out["keyframes"] = torch.zeros((B, H, 2, self.c.n_groups, 128), dtype=torch.int16,
                                           device=dev)
            out["state"] = torch.zeros((B, H, 2, 128), dtype=torch.float32, device=dev)
        if d.fmt == DKV_FMT_FP16:
            out["keyframes"] = torch.zeros((B, H, 2, cap, 128), dtype=torch.int16, device=dev)
        dkv_export_canonical(self.c, out.get("codes"), out.get("scales"), out.get("keyframes"),
                             out.get("state"), stream)
        return out

    def dequantize(self, stream=None):
        import torch
        d = self.desc
        out = torch.zeros((d.batch, d.n_kv_heads, 2, d.max_ctx, 128), dtype=torch.float32,
                          device=self.device)
        dkv_dequantize(self.c, out, stream)
        return out

    def device_status(self, stream=None) -> int:
        return dkv_get_device_status(self.c, stream)
