"""The C ABI: the library loads, exports every function the header declares, its
argument structure matches the header, and invalid arguments are rejected on the
host before any device work (so these tests need no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from linear_lsh_sketch_race_b200 import race_attn as ra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "race_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(race_[a-z_0-9]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = ra.load()
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(ra.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", ra.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (race_\w+)", out))
    assert set(names) <= exported


def test_args_struct_matches_header(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(r'''
#include <stdio.h>
#include <stddef.h>
#include "race_attn.h"
int main(void) {
  printf("%zu", sizeof(race_args_t));
#define F(m) printf(" %zu", offsetof(race_args_t, m));
  F(N) F(H) F(d) F(L) F(P) F(tau) F(causal) F(dtype) F(out_dtype) F(chunk)
  F(workspace) F(workspace_bytes) F(den) F(impl) F(grad_dtype) F(w_per_head)
  printf("\n");
  return 0;
}
''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    vals = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(ra.RaceArgs)
    fields = [f[0] for f in ra.RaceArgs._fields_]
    for name, off in zip(fields, vals[1:]):
        assert getattr(ra.RaceArgs, name).offset == off, name


def test_status_strings_and_version():
    for s in range(6):
        assert ra.race_status_string(s).startswith("RACE_")
    assert "unknown" in ra.race_status_string(99)
    assert ra.race_version() >= 100


def _args(**kw):
    a = ra.race_args_init(1024, 2, 64, 4, 4, 0.5, 1)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_args_init_defaults():
    a = _args()
    assert (a.N, a.H, a.d, a.L, a.P, a.causal) == (1024, 2, 64, 4, 4, 1)
    assert a.dtype == ra.RACE_BF16 and a.out_dtype == ra.RACE_BF16
    assert a.impl == ra.RACE_IMPL_AUTO and a.chunk == 0 and not a.workspace and not a.den
    assert a.grad_dtype == ra.RACE_BF16 and a.w_per_head == 0


@pytest.mark.parametrize("field,value,status", [
    ("N", 0, ra.RACE_ERR_INVALID_ARG),
    ("H", 0, ra.RACE_ERR_INVALID_ARG),
    ("L", 0, ra.RACE_ERR_INVALID_ARG),
    ("P", 0, ra.RACE_ERR_INVALID_ARG),
    ("P", 9, ra.RACE_ERR_INVALID_ARG),
    ("tau", 0.0, ra.RACE_ERR_INVALID_ARG),
    ("tau", -1.0, ra.RACE_ERR_INVALID_ARG),
    ("tau", float("nan"), ra.RACE_ERR_INVALID_ARG),
    ("tau", float("inf"), ra.RACE_ERR_INVALID_ARG),
    ("causal", 2, ra.RACE_ERR_INVALID_ARG),
    ("dtype", 7, ra.RACE_ERR_INVALID_ARG),
    ("impl", 5, ra.RACE_ERR_INVALID_ARG),
    ("chunk", -64, ra.RACE_ERR_INVALID_ARG),
    ("chunk", 100, ra.RACE_ERR_INVALID_ARG),
    ("grad_dtype", 3, ra.RACE_ERR_INVALID_ARG),
    ("w_per_head", 2, ra.RACE_ERR_INVALID_ARG),
    ("d", 32, ra.RACE_ERR_UNSUPPORTED),
    ("d", 128, ra.RACE_ERR_UNSUPPORTED),
])
def test_invalid_arguments_rejected_on_host(field, value, status):
    a = _args(**{field: value})
    n = ctypes.c_size_t(123)
    assert ra.load().race_workspace_size(ctypes.byref(a), 0, ctypes.byref(n)) == status
    assert n.value == 0
    # the forward rejects the same arguments before touching the device
    buf = 1 << 20   # any 16-byte-aligned non-null value: never dereferenced
    assert ra.load().race_forward_ex(buf, buf, buf, buf, buf, ctypes.byref(a), None) == status


def test_table_size_limit():
    a = _args(L=65, P=8)      # L * 2^P > 16384
    n = ctypes.c_size_t(0)
    assert ra.load().race_workspace_size(ctypes.byref(a), 0, ctypes.byref(n)) == \
        ra.RACE_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected():
    a = _args()
    lib = ra.load()
    good = 1 << 20
    assert lib.race_forward_ex(None, good, good, good, good, ctypes.byref(a), None) == \
        ra.RACE_ERR_INVALID_ARG
    assert lib.race_forward_ex(good + 2, good, good, good, good, ctypes.byref(a), None) == \
        ra.RACE_ERR_INVALID_ARG
    assert lib.race_backward_ex(*([good] * 9 + [None]), ctypes.byref(a), None) == \
        ra.RACE_ERR_INVALID_ARG
    assert lib.race_hash(good, good, good + 8, ctypes.byref(a), None) == \
        ra.RACE_ERR_INVALID_ARG
    assert lib.race_forward_ex(good, good, good, good, good, None, None) == \
        ra.RACE_ERR_INVALID_ARG


def test_workspace_size_queries():
    a = _args(N=4096, H=2, L=4, P=4)
    fw = ra.race_workspace_size(a, False)
    bw = ra.race_workspace_size(a, True)
    assert fw > 0 and bw >= fw
    # scratch grows linearly with N for a fixed head count
    a2 = _args(N=8192, H=2, L=4, P=4)
    assert ra.race_workspace_size(a2, True) > bw
    with pytest.raises(ra.RaceError):
        ra.race_workspace_size(_args(d=48), False)
    n = ctypes.c_size_t(0)
    assert ra.load().race_workspace_size(ctypes.byref(a), 0, None) == ra.RACE_ERR_INVALID_ARG


def test_too_small_caller_workspace_rejected():
    a = _args(N=4096, H=2, L=4, P=4)
    need = ra.race_workspace_size(a, False)
    a.workspace = 1 << 20
    a.workspace_bytes = need - 1
    good = 1 << 20
    assert ra.load().race_forward_ex(good, good, good, good, good, ctypes.byref(a), None) == \
        ra.RACE_ERR_WORKSPACE
