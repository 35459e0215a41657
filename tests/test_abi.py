"""The C ABI on the host: the library loads, exports every entry point that
include/dmuon.h declares, and rejects bad arguments before touching the GPU."""
import ctypes
import math
import re
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "dmuon.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dmuon_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("dmuon_step", "dmuon_step_ex", "dmuon_compute_update", "dmuon_cache_save",
                 "dmuon_cache_load", "dmuon_set_workspace", "dmuon_last_error"):
        assert must in names


def test_every_declared_symbol_is_exported(dmuon_lib):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", str(dmuon_lib.LIB_PATH)], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dmuon_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(dmuon_lib.EXPORTS) == set(names)
    for n in names:
        assert hasattr(dmuon_lib.lib, n)


def test_library_links_no_torch(dmuon_lib):
    out = subprocess.run(["ldd", str(dmuon_lib.LIB_PATH)], capture_output=True, text=True).stdout
    assert "torch" not in out and "libcudart" not in out  # runtime linked statically


def test_version_and_defaults(dmuon_lib):
    assert dmuon_lib.dmuon_version() == 1
    o = dmuon_lib.options()
    assert o.mom_dtype == dmuon_lib.DMUON_F32 and o.nesterov == 1 and o.variant == 0
    assert math.isclose(o.eps, 1e-7, rel_tol=1e-6)
    assert (round(o.ns_a, 4), round(o.ns_b, 4), round(o.ns_c, 4)) == (3.4445, -4.775, 2.0315)


def _call_step(lib, count=1, shapes=(4, 8), lr=0.02, wd=0.1, mu=0.95, steps=5, opts=None, nullp=False):
    P = (ctypes.c_void_p * 1)(0x1000)
    sh = (ctypes.c_int64 * 2)(*shapes)
    return lib.lib.dmuon_step_ex(None if nullp else P, P, P, sh, count, lr, wd, mu, steps,
                                 ctypes.byref(opts) if opts is not None else None, None)


def test_host_validation_rejects_before_any_launch(dmuon_lib):
    L = dmuon_lib
    assert _call_step(L, count=0) == L.DMUON_OK
    assert _call_step(L, count=-1) == L.DMUON_ERR_INVALID
    assert _call_step(L, steps=17) == L.DMUON_ERR_INVALID
    assert _call_step(L, steps=-1) == L.DMUON_ERR_INVALID
    assert _call_step(L, lr=float("nan")) == L.DMUON_ERR_INVALID
    assert _call_step(L, mu=float("inf")) == L.DMUON_ERR_INVALID
    assert _call_step(L, shapes=(0, 8)) == L.DMUON_ERR_INVALID
    assert _call_step(L, shapes=(8, -3)) == L.DMUON_ERR_INVALID
    assert _call_step(L, nullp=True) == L.DMUON_ERR_INVALID
    assert "NULL" in L.last_error() or "null" in L.last_error()
    o = L.options(L.DMUON_BF16, L.DMUON_F32)
    assert _call_step(L, opts=o) == L.DMUON_ERR_DTYPE
    o = L.options()
    o.mom_dtype = L.DMUON_BF16
    assert _call_step(L, opts=o) == L.DMUON_ERR_DTYPE
    o = L.options()
    o.variant = 9
    assert _call_step(L, opts=o) == L.DMUON_ERR_INVALID
    # the size limits: a side above 2^20, or more than 2^31 elements in one matrix
    assert _call_step(L, shapes=((1 << 20) + 1, 8)) == L.DMUON_ERR_INVALID
    assert _call_step(L, shapes=(8, (1 << 20) + 1)) == L.DMUON_ERR_INVALID
    assert _call_step(L, shapes=(1 << 16, (1 << 15) + 1)) == L.DMUON_ERR_INVALID
    assert "too large" in L.last_error()


def test_workspace_size_is_host_only_and_monotone(dmuon_lib):
    a = dmuon_lib.dmuon_workspace_size([(1024, 1024)] * 4)
    b = dmuon_lib.dmuon_workspace_size([(1024, 1024)] * 8)
    c = dmuon_lib.dmuon_workspace_size([(4096, 14336)])
    assert 0 < a < b < c
    # tall and wide need the same scratch (the iterate is always the wide one)
    assert dmuon_lib.dmuon_workspace_size([(300, 100)]) == dmuon_lib.dmuon_workspace_size([(100, 300)])


def test_gemm_argument_checks(dmuon_lib):
    L = dmuon_lib
    g = L.lib.dmuon_gemm_bf16
    assert g(None, 8, 64, None, 8, 64, 1, None, 0, 0, None, 8, 64, 8, 8, 8, 1, 1.0, 0.0, 0, 0, None) == L.DMUON_ERR_INVALID
    # lda not a multiple of 8
    assert g(16, 12, 0, 16, 8, 0, 1, None, 0, 0, 16, 8, 0, 8, 8, 8, 1, 1.0, 0.0, 0, 0, None) == L.DMUON_ERR_INVALID
    # unknown tile code
    assert g(16, 8, 0, 16, 8, 0, 1, None, 0, 0, 16, 8, 0, 8, 8, 8, 1, 1.0, 0.0, 96, 0, None) == L.DMUON_ERR_INVALID
    # symmetric output needs a square result
    assert g(16, 8, 0, 16, 8, 0, 1, None, 0, 0, 16, 16, 0, 8, 16, 8, 1, 1.0, 0.0, 0, 1, None) == L.DMUON_ERR_INVALID


def test_set_workspace_alignment(dmuon_lib):
    L = dmuon_lib
    assert L.lib.dmuon_set_workspace(ctypes.c_void_p(0x1001), 4096) == L.DMUON_ERR_INVALID
    assert L.lib.dmuon_set_workspace(None, 0) == L.DMUON_OK


def test_header_compiles_and_links_as_plain_c(dmuon_lib, tmp_path):
    """A C99 program includes include/dmuon.h, links libdmuon.so and calls
    entry points that need no GPU: the boundary is usable without C++ or
    Python."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "abi_check.c"
    src.write_text(r'''
#include <stdio.h>
#include "dmuon.h"
int main(void) {
  dmuon_options o;
  dmuon_options_init(&o);
  if (dmuon_version() != 1 || o.variant != DMUON_VARIANT_AUTO || o.mom_dtype != DMUON_F32) return 1;
  /* count 0 is a no-op; a null pointer array is rejected before any launch */
  if (dmuon_step(NULL, NULL, NULL, NULL, 0, 0.02f, 0.1f, 0.95f, 5, NULL) != 0) return 2;
  int64_t shape[2] = {4, 4};
  int rc = dmuon_step(NULL, NULL, NULL, shape, 1, 0.02f, 0.1f, 0.95f, 5, NULL);
  if (rc != DMUON_ERR_INVALID) return 3;
  printf("%d %s\n", rc, dmuon_last_error());
  return 0;
}
''')
    lib = Path(dmuon_lib.LIB_PATH)
    exe = tmp_path / "abi_check"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", f"-I{ROOT / 'include'}", str(src), "-o", str(exe),
                    f"-L{lib.parent}", "-ldmuon", f"-Wl,-rpath,{lib.parent}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith(str(dmuon_lib.DMUON_ERR_INVALID))
