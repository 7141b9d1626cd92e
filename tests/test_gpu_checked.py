"""The GPU parity suite on the bounds-checked build.

``libdkv_checked.so`` is the library compiled with DKV_CHECKED=1. Every
computed global memory range is tested against the buffer it must lie in:
- bulk-copy sources and destinations, partial records, handoffs and records
  of groups entered midway (against the workspace size);
- q rows and output rows;
- encoder and fused-append reads and writes of inputs, records and state.

A range outside its buffer sets DKV_DEV_BOUNDS in the device status word, and
the access is skipped. No GPU fault is caused or needed: the check runs before
the access.

The parity tests assert the status word is 0 after their launches and compare
with the oracle. So running them again on the checked build, in a subprocess
that loads it (DKV_LIBRARY=checked), shows that no kernel computes an
out-of-range address on those shapes: tiny, ragged, partial groups, every kf
class, paged, multi-query, fused, noalloc, and the full-size workloads.
"""
import os
import subprocess
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu
ROOT = Path(__file__).resolve().parent.parent

# every GPU parity file but this one (and the long stress sweep, whose shapes
# the edge-case and decode tests already cover)
FILES = ["test_gpu_encode.py", "test_gpu_decode.py", "test_gpu_edge_cases.py",
         "test_gpu_paged.py", "test_gpu_multiquery.py", "test_gpu_fused.py", "test_gpu_lr.py",
         "test_gpu_fullsize.py", "test_zz_no_alloc.py"]


def test_gpu_suite_on_checked_build():
    lib = ROOT / "delta_quantized_kv_b200" / "_lib" / "libdkv_checked.so"
    assert lib.exists(), "build() makes libdkv_checked.so beside libdkv.so"
    env = dict(os.environ, DKV_LIBRARY="checked")
    probe = subprocess.run(
        [sys.executable, "-c",
         "import delta_quantized_kv_b200 as d, ctypes; l = d.load(); print(l._name)"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert probe.returncode == 0, probe.stderr[-2000:]
    assert probe.stdout.strip().endswith("libdkv_checked.so"), probe.stdout
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        *[str(ROOT / "tests" / f) for f in FILES]],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=3000)
    tail = (r.stdout + r.stderr)[-3000:]
    print(tail)
    assert r.returncode == 0, tail


_SHRUNK = r"""
import sys
sys.path.insert(0, ".")
import torch
import delta_quantized_kv_b200 as d
import synthetic as S
w = S.WORKLOADS["llama3_8b_layer"].with_(B=2, T=200)
K, V = S.gen_kv(w)
c = d.Cache(2, w.Hkv, 200, "delta", kf=32)
c.encode(K.cuda(), V.cuda())
q = S.gen_q(w).cuda()
ref = c.decode_attn(q, 0.088)
torch.cuda.synchronize()
s0 = c.device_status()
d.dkv_debug_set_fault(2)
bad = c.decode_attn(q, 0.088)
torch.cuda.synchronize()
s1 = c.device_status()
d.dkv_debug_set_fault(0)
again = c.decode_attn(q, 0.088)
torch.cuda.synchronize()
s2 = c.device_status()
print("STATUS", s0, s1, s2, int(torch.equal(again, ref)), int(torch.equal(bad, ref)))
"""


@pytest.mark.parametrize("checked", [True, False])
def test_bounds_check_catches_a_short_workspace(checked):
    """Fault mode 2 declares the workspace two records short of what the
    split kernel writes (the buffer itself is full size).
    - The checked build must flag DKV_DEV_BOUNDS (0x20), skip those writes, and
      decode correctly again once the mode is off.
    - The normal build has no checks and must not notice."""
    env = dict(os.environ)
    if checked:
        env["DKV_LIBRARY"] = "checked"
    else:
        env.pop("DKV_LIBRARY", None)
    r = subprocess.run([sys.executable, "-c", _SHRUNK], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, (r.stdout + r.stderr)[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("STATUS")][-1]
    s0, s1, s2, again_eq, bad_eq = map(int, line.split()[1:])
    assert s0 == 0 and s2 == 0 and again_eq == 1, line
    if checked:
        assert s1 & 0x20, line              # DKV_DEV_BOUNDS
    else:
        assert s1 == 0 and bad_eq == 1, line
