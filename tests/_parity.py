"""Helpers shared by the GPU parity tests (comparison only; no method
arithmetic)."""
import numpy as np

# Attention tolerance: max over channels of |o - o_ref| divided by max over
# channels of |o_ref|, per (batch, query head) row.
ATTN_TOL = 2e-3


def row_rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.abs(got - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return np.where(den > 0, num / np.maximum(den, 1e-300), num)


def oracle_fields(orc, fmt, x, kf, cap):
    """Oracle's stored fields of one [len, D] tensor, padded to capacity."""
    x = np.asarray(x, dtype=np.float32)
    L, D = x.shape
    if fmt == "delta":
        s = orc.delta_encode(x, kf, cap=cap)
        return {"codes": s.codes, "scales": s.scales, "keyframes": s.kfr, "state": s.state}
    if fmt == "q4":
        sc, co, _ = orc.q4_encode(x)
        codes = np.zeros((cap, D), np.uint8); codes[:L] = co
        scales = np.zeros((cap, D // 32), np.uint16); scales[:L] = sc
        return {"codes": codes, "scales": scales}
    bits, _ = orc.f16_encode(x)
    kfr = np.zeros((cap, D), np.uint16); kfr[:L] = bits
    return {"keyframes": kfr}


def export_np(cache):
    ex = cache.export()
    out = {}
    for k, v in ex.items():
        a = v.cpu().numpy()
        if a.dtype == np.int16:
            a = a.view(np.uint16)
        out[k] = a
    return out


def assert_fields_equal(orc, cache, fmt, K, V, lens, kf, cap):
    """Every stored field of every (batch, kv head, tensor) sequence of the
    cache equals the oracle's encoding of the same tokens, bit for bit."""
    ex = export_np(cache)
    B, H = K.shape[0], K.shape[1]
    for b in range(B):
        for h in range(H):
            for t, X in enumerate((K, V)):
                x = np.asarray(X[b, h, :lens[b]], dtype=np.float32)
                ref = oracle_fields(orc, fmt, x, kf, cap)
                for k, r in ref.items():
                    got = ex[k][b, h, t]
                    if k == "keyframes" and fmt == "delta":
                        got = got[: r.shape[0]]
                    if k == "state":
                        if lens[b] == 0:
                            continue
                        assert np.array_equal(got.view(np.uint32), r.view(np.uint32)), \
                            (b, h, t, k)
                    else:
                        bad = np.argwhere(got != r)
                        assert bad.size == 0, (fmt, b, h, t, k, bad[:3].tolist(),
                                               [int(got[tuple(i)]) for i in bad[:3]],
                                               [int(r[tuple(i)]) for i in bad[:3]])
