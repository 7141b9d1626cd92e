"""Build the CUDA library ``_lib/libdkv.so`` for sm_100a with nvcc, and its
bounds-checked twin ``_lib/libdkv_checked.so`` (DKV_CHECKED=1: every computed
global memory range is tested against its buffer; tests load it with
DKV_LIBRARY=checked).

The libraries are compiled in-tree so the shared objects travel with the
source tree; nothing is installed into site-packages.
"""
from __future__ import annotations

import os
import shutil
import subprocess
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
OUT = PKG / "_lib" / "libdkv.so"
OUT_CHECKED = PKG / "_lib" / "libdkv_checked.so"
SOURCES = ["dkv_api.cu", "encode.cu", "decode.cu", "noalloc.cu", "lr_encode.cu", "lr_decode.cu"]
HEADERS = ["dkv_common.cuh", "dkv_internal.h"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not Path(cand).exists():
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libdkv")
    return cand


def stale(out: Path = OUT) -> bool:
    if not out.exists():
        return True
    t = out.stat().st_mtime
    deps = [CSRC / s for s in SOURCES + HEADERS] + [PKG.parent / "include" / "dkv.h"]
    return any(d.stat().st_mtime > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = True) -> Path:
    """Build the library (and, with checked, its bounds-checked twin, at the
    same time)."""
    if not checked:
        return _build_one(OUT, [], force, verbose)
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=2) as ex:
        jobs = [ex.submit(_build_one, OUT, [], force, verbose),
                ex.submit(_build_one, OUT_CHECKED, ["-DDKV_CHECKED=1"], force, verbose)]
        return [j.result() for j in jobs][0]


def _build_one(OUT: Path, extra: list, force: bool, verbose: bool) -> Path:
    """Compile every translation unit in parallel (one nvcc per file), then
    link the shared library; the result replaces the old one atomically."""
    if not force and not stale(OUT):
        return OUT
    from concurrent.futures import ThreadPoolExecutor
    import tempfile
    OUT.parent.mkdir(parents=True, exist_ok=True)
    nvcc = _nvcc()
    cflags = [f for f in NVCC_FLAGS if f != "-shared"] + extra
    with tempfile.TemporaryDirectory(prefix="dkv_build_") as tmpd:
        objs = [Path(tmpd) / (Path(s).stem + ".o") for s in SOURCES]

        def compile_one(i):
            cmd = [nvcc, *cflags, *(["-Xptxas", "-v"] if verbose else []), "-c",
                   str(CSRC / SOURCES[i]), "-o", str(objs[i])]
            return subprocess.run(cmd, capture_output=True, text=True)

        with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 1)) as ex:
            results = list(ex.map(compile_one, range(len(SOURCES))))
        for r in results:
            if verbose or r.returncode:
                print(r.stdout + r.stderr)
            if r.returncode:
                raise subprocess.CalledProcessError(r.returncode, r.args, r.stdout, r.stderr)
        tmp = OUT.with_name(f"{OUT.stem}.{os.getpid()}.tmp.so")
        subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                        "-o", str(tmp), *[str(o) for o in objs]], check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force=True))
