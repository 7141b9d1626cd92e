"""CPU-only checks of the C ABI: the library builds and loads, exports every
function include/dkv.h declares, sizes caches by the documented layout, and
rejects bad arguments before touching the GPU.  Also checks the host-side
arithmetic of the decode work split (which warp owns which unit, and the
partial-record slot of every (warp, sequence) pair)."""
import ctypes
import random
import re
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def dkv():
    from delta_quantized_kv_b200 import build
    build.build()
    import delta_quantized_kv_b200 as m
    m.load()
    return m


def _declared():
    text = (ROOT / "include" / "dkv.h").read_text()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(dkv_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(dkv):
    names = _declared()
    assert len(names) >= 13
    nm = subprocess.run(["nm", "-D", "--defined-only", str(dkv.LIB_PATH)], capture_output=True,
                        text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dkv_\w+)", nm))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(dkv.EXPORTS) <= exported


def test_abi_version_and_status_strings(dkv):
    hdr = (ROOT / "include" / "dkv.h").read_text()
    want = int(re.search(r"#define DKV_ABI_VERSION (\d+)", hdr).group(1))
    assert dkv.dkv_abi_version() == want
    for s in range(7):
        assert dkv.status_str(s) and dkv.status_str(s) != "unknown status"
    assert dkv.status_str(99) == "unknown status"


def _desc(dkv, B=16, H=8, D=128, kf=32, cap=32768, fmt=2):
    return dkv.dkv_cache_desc(B, H, D, kf, cap, fmt)


def test_cache_bytes_follow_the_layout(dkv):
    def expect(B, H, kf, cap, fmt):
        if fmt == 2:
            ng = -(-cap // kf)
            stride = ng * (512 + (kf - 1) * 144)
        elif fmt == 1:
            stride = cap * 144
        else:
            stride = cap * 512
        up = lambda x: (x + 255) // 256 * 256
        off_state = up(B * H * stride + 4096)
        off_seq = up(off_state + 2 * B * H * 2 * 128 * 4)
        off_hdr = up(off_seq + 4 * B)
        return up(off_hdr + 16), stride
    for (B, H, kf, cap, fmt) in [(16, 8, 32, 32768, 2), (1, 1, 1, 1, 2), (4, 8, 512, 131328, 2),
                                 (2, 3, 33, 1000, 2), (16, 8, 32, 32768, 1), (16, 8, 32, 32768, 0)]:
        tot, stride = expect(B, H, kf, cap, fmt)
        assert dkv.dkv_cache_bytes(_desc(dkv, B, H, 128, kf, cap, fmt)) == tot
    # the headline cache: 4976 B per 32-token group -> 155.5 B per token per kv head
    assert expect(16, 8, 32, 32768, 2)[1] * 16 * 8 == 652_214_272


@pytest.mark.parametrize("field,val", [("batch", 0), ("batch", 1025), ("n_kv_heads", 0),
                                       ("kf", 0), ("max_ctx", 0), ("fmt", 7)])
def test_invalid_descriptors_size_zero(dkv, field, val):
    d = _desc(dkv)
    setattr(d, field, val)
    assert dkv.dkv_cache_bytes(d) == 0


def test_head_dim_must_be_128(dkv):
    d = _desc(dkv, D=64)
    assert dkv.dkv_cache_bytes(d) == 0
    out = dkv.dkv_cache()
    s = dkv.load().dkv_cache_init(ctypes.byref(d), 4096, 1 << 30, ctypes.byref(out), None)
    assert s == dkv.DKV_EUNSUPPORTED


def test_init_rejects_bad_pointers_without_a_launch(dkv):
    lib = dkv.load()
    d = _desc(dkv, B=1, H=1, cap=64)
    out = dkv.dkv_cache()
    n = dkv.dkv_cache_bytes(d)
    assert lib.dkv_cache_init(ctypes.byref(d), None, n, ctypes.byref(out), None) == dkv.DKV_EINVAL
    assert lib.dkv_cache_init(ctypes.byref(d), 4096 + 16, n, ctypes.byref(out), None) == dkv.DKV_EALIGN
    assert lib.dkv_cache_init(ctypes.byref(d), 4096, n - 1, ctypes.byref(out), None) == dkv.DKV_ECAPACITY


def test_calls_on_an_invalid_cache_are_rejected(dkv):
    lib = dkv.load()
    c = dkv.dkv_cache()          # base == NULL
    assert lib.dkv_encode(ctypes.byref(c), 16, 16, 1, None, 8, None) == dkv.DKV_EINVAL
    assert lib.dkv_append(ctypes.byref(c), 16, 16, 1, 1, None) == dkv.DKV_EINVAL
    assert lib.dkv_decode_attn(ctypes.byref(c), 16, 1, 8, 1.0, 16, 16, 1 << 20, None) == dkv.DKV_EINVAL
    assert lib.dkv_dequantize(ctypes.byref(c), 16, None) == dkv.DKV_EINVAL
    assert lib.dkv_append_decode_attn(ctypes.byref(c), 16, 16, 1, 1, 16, 1, 8, 1.0, 16, 16,
                                      1 << 20, None) == dkv.DKV_EINVAL
    w = ctypes.c_int32(0)
    assert lib.dkv_get_device_status(ctypes.byref(c), ctypes.byref(w), None) == dkv.DKV_EINVAL


def test_noalloc_gives_invalid_caches_the_statuses_of_dkv_decode_attn(dkv):
    """The no-workspace decode validates the cache before it sizes the step,
    so a bad descriptor gets the same status as from dkv_decode_attn (and
    nothing touches the GPU)."""
    lib = dkv.load()
    for field, val, want in [("kf", 0, dkv.DKV_EINVAL), ("head_dim", 64, dkv.DKV_EUNSUPPORTED),
                             ("fmt", 9, dkv.DKV_EINVAL), ("batch", 0, dkv.DKV_EINVAL),
                             ("max_ctx", 0, dkv.DKV_EINVAL)]:
        c = dkv.dkv_cache()
        c.desc = _desc(dkv, B=2, H=2, cap=100)
        setattr(c.desc, field, val)
        c.base = 1 << 20
        c.bytes = 1 << 30
        got = lib.dkv_decode_attn_noalloc(ctypes.byref(c), 1 << 12, 1, 8, 1.0, 1 << 12, None)
        ref = lib.dkv_decode_attn(ctypes.byref(c), 1 << 12, 1, 8, 1.0, 1 << 12, 1 << 12,
                                  1 << 30, None)
        assert got == ref == want, (field, got, ref, want)
    c = dkv.dkv_cache()                                   # base == NULL
    assert lib.dkv_decode_attn_noalloc(ctypes.byref(c), 1 << 12, 1, 8, 1.0, 1 << 12,
                                       None) == dkv.DKV_EINVAL


def test_lr_decode_rejects_bad_arguments_on_host(dkv):
    """dkv_lr_decode_attn validates everything before any launch."""
    lib = dkv.load()
    A = 1 << 12
    t = dkv.dkv_lr_tensor(A, A, A, A)
    bad = dkv.dkv_lr_tensor(A, A + 2, A, A)
    nb = dkv.dkv_lr_decode_workspace_bytes(2, 2, 100, 8)
    assert nb > 0 and dkv.dkv_lr_decode_workspace_bytes(0, 2, 100, 8) == 0
    call = lambda K=t, V=t, B=2, H=2, T=100, s=8, m=2, q=A, qd=1, hq=8, sc=0.1, o=A, ws=A, wsb=nb: \
        lib.dkv_lr_decode_attn(ctypes.byref(K), ctypes.byref(V), B, H, T, s, m, None, q, qd, hq,
                               sc, o, ws, wsb, None)
    assert call(K=dkv.dkv_lr_tensor(0, A, A, A)) == dkv.DKV_EINVAL
    assert call(V=bad) == dkv.DKV_EALIGN
    assert call(m=0) == dkv.DKV_EINVAL and call(m=9) == dkv.DKV_EINVAL
    assert call(s=0) == dkv.DKV_EINVAL and call(T=0) == dkv.DKV_EINVAL
    assert call(hq=3) == dkv.DKV_EINVAL
    assert call(hq=18) == dkv.DKV_EUNSUPPORTED            # 9 query heads per kv head
    assert call(sc=0.0) == dkv.DKV_EINVAL and call(qd=7) == dkv.DKV_EINVAL
    assert call(q=A + 4) == dkv.DKV_EALIGN
    assert call(wsb=nb - 4) == dkv.DKV_ECAPACITY
    assert lib.dkv_lr_decode_attn(None, ctypes.byref(t), 2, 2, 100, 8, 2, None, A, 1, 8, 0.1,
                                  A, A, nb, None) == dkv.DKV_EINVAL


def test_division_check_rejects_bad_arguments(dkv):
    lib = dkv.load()
    assert lib.dkv_debug_division_check(None, 4, 1 << 12, None) == dkv.DKV_EINVAL
    assert lib.dkv_debug_division_check(1 << 12, 0, 1 << 12, None) == dkv.DKV_EINVAL
    assert lib.dkv_debug_division_check(1 << 12, 4, (1 << 12) + 8, None) == dkv.DKV_EALIGN


def test_bad_dtype_and_sizes_rejected_on_host(dkv):
    """A well-formed view whose arguments are wrong: nothing is launched."""
    lib = dkv.load()
    d = _desc(dkv, B=2, H=2, cap=100)
    n = dkv.dkv_cache_bytes(d)
    c = dkv.dkv_cache()
    c.desc = d
    c.base = 1 << 20
    c.bytes = n
    # replicate the layout the library computes (offsets must agree)
    up = lambda x: (x + 255) // 256 * 256
    ng = -(-100 // 32)
    c.seq_stride = ng * (512 + 31 * 144)
    c.rec_bytes = 512 + 31 * 144
    c.n_groups = ng
    c.off_state = up(4 * c.seq_stride + 4096)
    c.off_seqlen = up(c.off_state + 2 * 4 * 2 * 128 * 4)
    c.off_header = up(c.off_seqlen + 8)
    assert lib.dkv_encode(ctypes.byref(c), 1 << 12, 1 << 12, 9, None, 8, None) == dkv.DKV_EINVAL
    assert lib.dkv_encode(ctypes.byref(c), (1 << 12) + 2, 1 << 12, 1, None, 8, None) == dkv.DKV_EALIGN
    assert lib.dkv_encode(ctypes.byref(c), 1 << 12, 1 << 12, 1, None, 101, None) == dkv.DKV_ECAPACITY
    assert lib.dkv_append(ctypes.byref(c), 1 << 12, 1 << 12, 1, 0, None) == dkv.DKV_EINVAL
    # n_q_heads not a multiple of n_kv_heads
    assert lib.dkv_decode_attn(ctypes.byref(c), 1 << 12, 1, 3, 1.0, 1 << 12, 1 << 12, 1 << 30,
                               None) == dkv.DKV_EINVAL
    # fused append + decode: K/V dtype, alignment, token count, heads, scale
    fused = lambda kvd=1, k=1 << 12, n=1, hq=4, s=1.0: lib.dkv_append_decode_attn(
        ctypes.byref(c), k, 1 << 12, kvd, n, 1 << 12, 1, hq, s, 1 << 12, 1 << 12, 1 << 30, None)
    assert fused(kvd=9) == dkv.DKV_EINVAL
    assert fused(k=(1 << 12) + 2) == dkv.DKV_EALIGN
    assert fused(n=0) == dkv.DKV_EINVAL
    assert fused(n=257) == dkv.DKV_EINVAL
    assert fused(hq=3) == dkv.DKV_EINVAL
    assert fused(s=0.0) == dkv.DKV_EINVAL
    assert lib.dkv_append_decode_attn_merge(ctypes.byref(c), 1, 4, (1 << 12) + 4, 1 << 12,
                                            1 << 30, None) == dkv.DKV_EALIGN
    # only the delta format appends inside the decode (a well-formed Q4_0 view)
    c.desc.fmt = 1
    c.seq_stride, c.rec_bytes, c.n_groups = 100 * 144, 0, 0
    c.off_state = up(4 * c.seq_stride + 4096)
    c.off_seqlen = up(c.off_state + 2 * 4 * 2 * 128 * 4)
    c.off_header = up(c.off_seqlen + 8)
    c.bytes = dkv.dkv_cache_bytes(c.desc)
    assert fused() == dkv.DKV_EUNSUPPORTED


def test_lr_encode_rejects_bad_arguments_on_host(dkv):
    """dkv_lr_encode validates before any launch: pointers, dtype, sizes,
    stride, reference count (1..8) and 16-byte alignment."""
    lib = dkv.load()
    A = 1 << 20

    def call(X=A, dt=1, n=2, T=64, s=8, m=2, ref=A, kv=A, sc=A, co=A, xh=A):
        return lib.dkv_lr_encode(X, dt, n, T, s, m, ref, kv, sc, co, xh, None)
    assert call(X=None) == dkv.DKV_EINVAL
    assert call(co=None) == dkv.DKV_EINVAL
    assert call(dt=7) == dkv.DKV_EINVAL
    assert call(n=0) == dkv.DKV_EINVAL
    assert call(T=0) == dkv.DKV_EINVAL
    assert call(s=0) == dkv.DKV_EINVAL
    assert call(m=0) == dkv.DKV_EINVAL
    assert call(m=9) == dkv.DKV_EINVAL
    assert call(n=65536) == dkv.DKV_EINVAL
    assert call(n=60000, T=60000) == dkv.DKV_ECAPACITY
    assert call(X=A + 2) == dkv.DKV_EALIGN
    assert call(sc=A + 8) == dkv.DKV_EALIGN
    assert call(xh=A + 4) == dkv.DKV_EALIGN


# ---- the decode work split (restated from the kernel's range arithmetic) ----
def _start(w, NW, T):
    return (w * T) // NW


def _warp_of(x, NW, T):
    return ((x + 1) * NW - 1) // T


def test_work_split_covers_every_unit_once_and_slots_are_unique():
    rng = random.Random(5)
    for _ in range(300):
        nseq = rng.randint(1, 40)
        units = [rng.choice([0, 1, 2, 3, 7, 50, 1024]) for _ in range(nseq)]
        T = sum(units)
        if T == 0:
            continue
        NW = rng.choice([1, 3, 4, 37, 592, 1776])
        owner = {}
        for w in range(NW):
            for x in range(_start(w, NW, T), _start(w + 1, NW, T)):
                assert x not in owner
                owner[x] = w
        assert len(owner) == T
        for x in range(T):
            assert _warp_of(x, NW, T) == owner[x]
        # slots (warp + sequence) written by warps that touch a sequence
        starts = [0]
        for u in units:
            starts.append(starts[-1] + u)
        slots = {}
        for s in range(nseq):
            xs, xe = starts[s], starts[s + 1]
            if xs == xe:
                continue
            for w in range(_warp_of(xs, NW, T), _warp_of(xe - 1, NW, T) + 1):
                if _start(w, NW, T) >= _start(w + 1, NW, T):
                    continue
                slot = w + s
                assert slot not in slots, (slot, slots.get(slot), (w, s))
                slots[slot] = (w, s)
                assert slot < NW + nseq


def test_paged_sizes_and_argument_checks(dkv):
    """Paged cache (delta format): metadata and page sizes follow the record
    layout, and bad arguments are rejected on the host before any launch."""
    import ctypes
    d = _desc(dkv, B=4, H=8, kf=32, cap=4096)
    rec = 512 + 31 * 144
    assert dkv.dkv_page_bytes(d, 16) == -(-8 * 16 * rec // 256) * 256
    assert dkv.dkv_page_bytes(d, 0) == 0
    meta = dkv.dkv_cache_meta_bytes(d)
    # fp32 state [2][B][Hkv][2][128], seq_len[B], header: no data area
    assert 2 * 4 * 8 * 2 * 128 * 4 < meta < 2 * 4 * 8 * 2 * 128 * 4 + 4096
    assert dkv.dkv_cache_meta_bytes(_desc(dkv, fmt=1)) == 0          # Q4_0 is not paged
    lib = dkv.load()
    out = dkv.dkv_cache()
    A = 1 << 20                                                          # 256-aligned fake addresses
    # too few block-table columns for max_ctx (4096 / 32 = 128 groups, 16 per page -> 8)
    assert lib.dkv_cache_init_paged(ctypes.byref(d), 16, A, 64, A, 7, A, meta, ctypes.byref(out),
                                    None) == dkv.DKV_EINVAL
    # misaligned pool, meta too small, page_groups < 1, comparator format
    assert lib.dkv_cache_init_paged(ctypes.byref(d), 16, A + 16, 64, A, 8, A, meta,
                                    ctypes.byref(out), None) == dkv.DKV_EALIGN
    assert lib.dkv_cache_init_paged(ctypes.byref(d), 16, A, 64, A, 8, A, meta - 1,
                                    ctypes.byref(out), None) == dkv.DKV_ECAPACITY
    assert lib.dkv_cache_init_paged(ctypes.byref(d), 0, A, 64, A, 8, A, meta, ctypes.byref(out),
                                    None) == dkv.DKV_EINVAL
    dq = _desc(dkv, B=4, H=8, cap=4096, fmt=1)
    assert lib.dkv_cache_init_paged(ctypes.byref(dq), 16, A, 64, A, 8, A, meta,
                                    ctypes.byref(out), None) == dkv.DKV_EUNSUPPORTED


# ---- fused append: which warp stores which new token (restated walk) -------
def _append_walk(units_of_seq, nvs, r0, r1, lens, n, kf, cap, pre, nhg):
    """The groups (b, vs, g) a warp with range [r0, r1) stores new tokens of, in
    its two phases (units [0, pre) of the range before its first copies, the
    rest after), and the (b, kv head) states it writes."""
    stores, states = [], []
    # locate the range's first unit
    x, b = 0, 0
    while b < len(lens) and x + nvs * units_of_seq[b] <= r0:
        x += nvs * units_of_seq[b]
        b += 1
    r = r0 - x
    vs, g0, ub = r // units_of_seq[b], r % units_of_seq[b], units_of_seq[b]
    for lo, hi in ((0, min(pre, r1 - r0)), (pre, r1 - r0)):
        if lo >= hi:
            continue
        bb, vv, gg, uu, off = b, vs, g0, ub, 0
        while off < hi:
            seg = uu - gg
            if off + seg > lo:
                ga = gg + max(0, lo - off)
                gb = gg + min(hi, off + seg) - off - 1
                L = lens[bb]
                if 0 <= L <= cap and L + n <= cap:
                    first = max(ga, L // kf)
                    for g in range(first, gb + 1):
                        stores.append((bb, vv, g))
                    if first <= gb and gb == uu - 1 and vv % nhg == 0:
                        states.append((bb, vv // nhg))
            off += seg
            if off >= hi:
                break
            gg = 0
            vv += 1
            if vv == nvs:
                vv = 0
                while True:
                    bb += 1
                    if bb >= len(lens):
                        break
                    uu = units_of_seq[bb]
                    if uu:
                        break
                if bb >= len(lens):
                    break
    return stores, states


def test_fused_append_walk_stores_every_new_group_once_per_owner():
    """Every group holding new tokens is stored by the warp that owns it (so
    that warp's own copy reads it after its own stores), no warp stores a group
    it does not own, and each (batch entry, kv head) that takes tokens has
    exactly one state writer."""
    rng = random.Random(11)
    for _ in range(300):
        B, Hkv, nhg = rng.randint(1, 5), rng.randint(1, 3), rng.choice([1, 1, 2, 3])
        kf, n = rng.choice([1, 3, 16, 32, 64]), rng.choice([1, 1, 2, 5])
        cap = rng.choice([40, 100, 300])
        lens = [rng.choice([0, 1, 31, 32, 33, 64, cap - n, cap - n + 1, cap, -1, cap + 1])
                for _ in range(B)]
        nvs = Hkv * nhg
        dec = [(L + n if 0 <= L <= cap and L + n <= cap else (L if 0 <= L <= cap else 0))
               for L in lens]
        units = [-(-d // kf) if d > 0 else 0 for d in dec]
        T = sum(nvs * u for u in units)
        if T == 0:
            continue
        NW = rng.choice([1, 2, 7, 64, 300])
        pre = rng.choice([1, 2])
        owner = {}
        x = 0
        for b in range(B):
            for vs in range(nvs):
                for g in range(units[b]):
                    owner[(b, vs, g)] = ((x + 1) * NW - 1) // T
                    x += 1
        stored, writers = {}, {}
        for w in range(NW):
            r0, r1 = (w * T) // NW, ((w + 1) * T) // NW
            if r0 >= r1:
                continue
            st, sw = _append_walk(units, nvs, r0, r1, lens, n, kf, cap, pre, nhg)
            for key in st:
                assert owner[key] == w, (key, w)
                stored[key] = stored.get(key, 0) + 1
            for key in sw:
                writers[key] = writers.get(key, 0) + 1
        for b, L in enumerate(lens):
            takes = 0 <= L <= cap and L + n <= cap
            for vs in range(nvs):
                new_groups = range(L // kf, units[b]) if takes else range(0)
                for g in new_groups:
                    assert stored.get((b, vs, g)) == 1, (b, vs, g, lens, n, kf)
            for kvh in range(Hkv):
                assert writers.get((b, kvh), 0) == (1 if takes else 0), (b, kvh, lens)
        assert all(k[2] >= max(0, lens[k[0]]) // kf for k in stored)
