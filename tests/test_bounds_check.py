"""The bounds-checked build (-DRACE_BOUNDS_CHECK).

* Host: the index predicate the kernels call (csrc/bounds.h, plain C++) compiled with the
  host compiler and run on edge cases: negative indices, the last valid index, one past
  it, empty ranges and indices beyond 2^31 and 2^63.
* Host: the library compiles with the flag and exports the same entry points (the build
  is a compile of the whole library, about a minute; it runs once, shared by the tests).
* GPU: the checked library gives the same outputs as the normal one on the hard-hash and
  the pipelined backward paths, with no bounds bit raised.
"""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_lsh_sketch_race_b200", "csrc")

PROBE = r"""
#include <stdio.h>
#include "bounds.h"
int main() {
  struct { long long i, n; int want; } cases[] = {
    {0, 1, 1}, {0, 0, 0}, {-1, 10, 0}, {9, 10, 1}, {10, 10, 0}, {5, -3, 0},
    {(1LL << 31) + 5, (1LL << 32), 1}, {(1LL << 32), (1LL << 32), 0},
    {-(1LL << 62), (1LL << 62), 0}, {(long long)0x7fffffffffffffffLL, 5, 0},
    {(long long)0x7ffffffffffffffeLL, (long long)0x7fffffffffffffffLL, 1},
  };
  int bad = 0;
  for (unsigned c = 0; c < sizeof(cases) / sizeof(cases[0]); ++c)
    if ((int)race::index_in_range(cases[c].i, cases[c].n) != cases[c].want) {
      printf("case %u wrong\n", c);
      ++bad;
    }
  printf("%d\n", bad);
  return bad;
}
"""


def test_index_predicate_on_the_host(tmp_path):
    src = tmp_path / "probe.cpp"
    src.write_text(PROBE)
    exe = tmp_path / "probe"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout


@pytest.fixture(scope="module")
def checked_lib():
    sys.path.insert(0, ROOT)
    from linear_lsh_sketch_race_b200 import build as b
    return b.build(bounds_check=True)


def test_checked_library_builds_and_exports_the_entry_points(checked_lib):
    sys.path.insert(0, ROOT)
    from linear_lsh_sketch_race_b200 import race_attn as ra
    lib = ctypes.CDLL(checked_lib)
    for name in ra.EXPORTED:
        assert hasattr(lib, name), name


GPU_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from linear_lsh_sketch_race_b200 import race_attn as ra
from linear_lsh_sketch_race_b200 import inputs as I

ra.load(sys.argv[2])
wl = I.Workload("bc", H=2, N=1500, d=64, L=2, P=8, tau=0.5, causal=True, dtype="bf16",
                seed=3, backward=True)
x = {k: v.to("cuda") for k, v in I.make_inputs(wl, "cpu").items()}
out = ra.forward(x["q"], x["k"], x["v"], x["W"], wl.tau, True, out_dtype=torch.float32)
grads = ra.backward(x["q"], x["k"], x["v"], x["W"], wl.tau, True, out, x["dout"],
                    impl="tensor", grad_dtype=torch.float32)
ho, cnt = ra.hard_forward(x["q"], x["k"], x["v"], x["W"], True, out_dtype=torch.float32)
torch.cuda.synchronize()
res = {n: t.double().cpu().numpy() for n, t in
       zip(("out", "dq", "dk", "dv", "dW", "hard"), (out, *grads, ho))}
res["cnt"] = cnt.cpu().numpy()
res["status"] = np.array(ra.race_device_status())
np.savez(sys.argv[3], **res)
"""


@pytest.mark.gpu
def test_checked_library_matches_the_normal_library(checked_lib, tmp_path):
    import numpy as np
    from linear_lsh_sketch_race_b200 import build as b
    script = tmp_path / "run.py"
    script.write_text(GPU_SCRIPT)
    res = []
    for i, lib in enumerate((b.LIB, checked_lib)):   # one process per library
        dst = tmp_path / f"r{i}.npz"
        r = subprocess.run([sys.executable, str(script), ROOT, lib, str(dst)],
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout + r.stderr
        res.append(np.load(dst))
    a, c = res
    assert int(a["status"]) == 0 and int(c["status"]) == 0
    assert (a["cnt"] == c["cnt"]).all()
    for n in ("out", "dq", "dk", "dv", "dW", "hard"):
        # the same kernels: float32 sums into shared accumulators may differ in order
        assert np.abs(a[n] - c[n]).max() <= 1e-5 * max(1.0, np.abs(a[n]).max()), n
