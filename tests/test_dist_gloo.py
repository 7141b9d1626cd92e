"""Multi-rank host logic of bench.py on CPU with the gloo backend
(world size 2): the timing reduction takes the max over ranks, the barrier
completes, and only rank 0 runs the reference arm."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(1.5 + rank, world)
        r, w, l = bench.dist_env()
        q.put((rank, got, r, w, l))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_env_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]
    assert [(r[2], r[3], r[4]) for r in res] == [(0, 2, 0), (1, 2, 1)]


def test_reference_arm_other_ranks_exit_silently(monkeypatch):
    sys.path.insert(0, str(ROOT))
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert rc == 0 and buf.getvalue() == ""


def test_kv_bytes_model():
    sys.path.insert(0, str(ROOT))
    import bench
    # headline cache: 4,194,304 (token, kv head) units at 155.5 B each
    assert bench.kv_bytes("delta", [32768] * 16, 8, 32) == 652_214_272
    assert bench.kv_bytes("q4", [32768] * 16, 8, 32) == 603_979_776
    assert bench.kv_bytes("fp16", [32768] * 16, 8, 32) == 2_147_483_648
    # a partial last group still pays a whole keyframe
    assert bench.kv_bytes("delta", [33], 1, 32) == 2 * 512 + 31 * 144


def test_long_range_quality_report_logic():
    """bench.lr_quality's bookkeeping (cases, keys, ratios), driven on the CPU
    by the oracle in place of the GPU encoder and caches: the long-range
    encoding must beat plain Q4_0 on the window-repeat generator, where far
    repeats are what the strided references exploit."""
    import numpy as np
    import torch
    import bench
    import oracle

    def enc(X, s, m):
        return torch.stack([torch.from_numpy(oracle.lr_encode(X[i].float().numpy(), s, m)["xhat"])
                            for i in range(X.shape[0])])

    def recon(fmt, K, V, kf):
        f = lambda A: torch.stack([torch.from_numpy(
            oracle.encode_cache(fmt, A[i].float().numpy(), kf)["xhat"]) for i in range(A.shape[0])])
        return f(K), f(V)

    saved = bench.LR_CASES
    bench.LR_CASES = [("batched_decode", "repeat", 256)]
    try:
        rep = bench.lr_quality("cpu", enc, recon)
    finally:
        bench.LR_CASES = saved
    (key, row), = rep.items()
    assert key == "batched_decode_repeat_T256_stride32"
    assert set(row) == {"lr_1_ref", "lr_4_ref", "delta", "q4"}
    assert all(np.isfinite(v) and v >= 0 for v in row.values())
    assert row["lr_1_ref"] < 0.1 * row["q4"]


def test_quality_report_arithmetic_against_numpy():
    """bench.quality_report's error figures, with the oracle's reconstruction
    standing in for the GPU caches, against the same quantities written out in
    numpy float64: relative MSE sum (x^ - x)^2 / sum x^2 over K and V;
    D_K = sum (q.k^ - q.k)^2 / sum (q.k)^2; D_V = |P V^ - P V|^2 / |P V|^2 with
    P the softmax of the scaled exact scores."""
    import numpy as np
    import torch
    import bench
    import oracle
    import synthetic as S

    def recon(fmt, K, V, kf):
        f = lambda A: torch.stack([torch.from_numpy(
            oracle.encode_cache(fmt, A[i].float().numpy(), kf)["xhat"]) for i in range(A.shape[0])])
        return f(K), f(V)

    cases = [("tiny", None, None), ("llama3_8b_layer", None, None)]
    rep = bench.quality_report("cpu", max_batch=1, recon=recon, cases=cases)
    for name, _, _ in cases:
        w = S.WORKLOADS[name]
        K, V = S.gen_kv_one(w, 0, w.T)
        G = w.Hq // w.Hkv
        q = S.gen_q(w)[0].double().numpy().reshape(w.Hkv, G, w.D)
        x = np.concatenate([K.double().numpy(), V.double().numpy()])
        for fmt in ("delta", "q4", "fp16"):
            kh, vh = (t.double().numpy() for t in recon(fmt, K, V, w.kf))
            xh = np.concatenate([kh, vh])
            rel = ((xh - x) ** 2).sum() / (x ** 2).sum()
            s_ref = np.einsum("hgd,htd->hgt", q, K.double().numpy())
            s_hat = np.einsum("hgd,htd->hgt", q, kh)
            z = s_ref / np.sqrt(w.D)
            P = np.exp(z - z.max(axis=-1, keepdims=True))
            P /= P.sum(axis=-1, keepdims=True)
            o_ref = np.einsum("hgt,htd->hgd", P, V.double().numpy())
            o_hat = np.einsum("hgt,htd->hgd", P, vh)
            dk = ((s_hat - s_ref) ** 2).sum() / (s_ref ** 2).sum()
            dv = ((o_hat - o_ref) ** 2).sum() / (o_ref ** 2).sum()
            got = rep[name][fmt]
            assert got["rel_mse"] == pytest.approx(rel, rel=1e-5, abs=1e-12), (name, fmt)
            assert got["D_K"] == pytest.approx(dk, rel=2e-2, abs=1e-12), (name, fmt)
            assert got["D_V"] == pytest.approx(dv, rel=2e-2, abs=1e-12), (name, fmt)
        assert rep[name]["entries"] == 1
        assert rep[name]["delta"]["rel_mse"] < rep[name]["q4"]["rel_mse"]


def test_multi_gpu_runs_only_the_timed_step(monkeypatch):
    """Under torchrun with N > 1 replicas the untimed extras (other workloads,
    comparator formats, quality report) and the host-core oracle baseline are
    switched off, so rank 0 does not hold N GPUs alone; at N = 1 they stay on."""
    sys.path.insert(0, str(ROOT))
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    one = bench.parse_args([])
    assert one.cpu_baseline and one.comparators and one.configs
    monkeypatch.setenv("WORLD_SIZE", "2")
    two = bench.parse_args(["--steps", "7", "--warmup", "1"])
    assert not (two.cpu_baseline or two.comparators or two.configs)
    assert two.steps == 7 and two.warmup == 3      # at least 3 warm-up steps
