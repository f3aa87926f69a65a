"""CPU-side checks of the C-ABI library: it loads without a GPU, exports
every entry point the header declares, and rejects bad arguments on the host
before anything is launched. No compute call is made here."""
import ctypes
import os
import re

import pytest
import torch

import packed_variable_length_attn_b200 as va
from packed_variable_length_attn_b200 import build as va_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    va_build.build()
    return va.load_library()


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(varlen_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(lib):
    names = _declared()
    assert "varlen_attn_fwd" in names and "varlen_attn_fwd_f32" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(va.exported_symbols()) <= set(names) | set()
    assert set(names) <= set(va.exported_symbols())


def test_strerror_and_version(lib):
    for code in range(0, 12):
        assert va.strerror(code)
    assert va.strerror(999) == "unknown status"
    assert lib.varlen_attn_version() >= 100
    assert va.launches_per_call() == 2


def _call(lib, **kw):
    a = dict(q=16, k=16, v=16, cu_q=16, cu_k=16, batch=1, total_q=8, total_k=8, max_q=8, max_k=8,
             hq=2, hkv=2, d=64, scale=0.125, causal=1, bk=None, bp=None, sb=0, sh=0, sr=0, sc=0,
             out=16, lse=16, stream=None)
    a.update(kw)
    p = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.varlen_attn_fwd(p(a["q"]), p(a["k"]), p(a["v"]), p(a["cu_q"]), p(a["cu_k"]),
                               a["batch"], a["total_q"], a["total_k"], a["max_q"], a["max_k"],
                               a["hq"], a["hkv"], a["d"], a["scale"], a["causal"], p(a["bk"]),
                               p(a["bp"]), a["sb"], a["sh"], a["sr"], a["sc"], p(a["out"]),
                               p(a["lse"]), a["stream"])


def test_host_validation_codes(lib):
    # the pointer values are never dereferenced: validation fails first
    assert _call(lib, q=None) == 1
    assert _call(lib, cu_k=None) == 1
    assert _call(lib, k=None) == 1          # keys exist: k and v are required
    assert _call(lib, v=None) == 1
    if not torch.cuda.is_available():       # with no keys NULL k/v pass validation
        assert _call(lib, k=None, v=None, total_k=0, max_k=0) == 7
    assert _call(lib, batch=0) == 2
    assert _call(lib, hq=0) == 2
    assert _call(lib, total_q=-1) == 2
    assert _call(lib, hq=3, hkv=2) == 3
    assert _call(lib, d=96) == 4
    assert _call(lib, d=256) == 4
    assert _call(lib, q=24) == 5            # not 16-byte aligned
    assert _call(lib, out=8) == 5
    assert _call(lib, lse=18) == 5          # not 4-byte aligned
    assert _call(lib, bp=16, sc=-1) == 6
    assert _call(lib, total_q=1 << 30, hq=4, hkv=4) == 11


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU failure path")
def test_no_device_is_an_error_not_a_fallback(lib):
    # valid arguments on a machine without a GPU: a CUDA error code, no output
    assert _call(lib) == 7
    q = torch.zeros(8, 2, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 8], dtype=torch.int32)
    with pytest.raises(ValueError):
        va.varlen_attn_fwd(q, q, q, cu, cu, 8, 8)


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(va, "_lib", None)
    monkeypatch.setattr(va, "_LIB_PATH", "/nonexistent/libvarlen_attn.so")
    with pytest.raises(ImportError):
        va.load_library()


def test_helper_host_validation_codes(lib):
    p = ctypes.c_void_p
    # varlen_attn_fwd_ex: unknown flag bits are rejected before any device work
    assert lib.varlen_attn_fwd_ex(p(16), p(16), p(16), p(16), p(16), 1, 8, 8, 8, 8, 2, 2, 64,
                                  0.125, 1, None, None, 0, 0, 0, 0, 2, p(16), p(16), None) == 6
    assert lib.varlen_mask_to_seqlens(None, 2, 4, p(16), p(16), p(16), None) == 1
    assert lib.varlen_mask_to_seqlens(p(16), 0, 4, p(16), p(16), p(16), None) == 2
    assert lib.varlen_mask_to_seqlens(p(16), 2, 4, p(18), p(16), p(16), None) == 5
    assert lib.varlen_mask_to_seqlens(p(16), 1 << 16, 1 << 16, p(16), p(16), p(16), None) == 11
    for fn in (lib.varlen_gather_rows, lib.varlen_scatter_rows):
        assert fn(None, 4, 32, p(16), p(16), 1, p(16), 4, None) == 1
        assert fn(p(16), 4, 24, p(16), p(16), 1, p(16), 4, None) == 2   # rows not 16-byte units
        assert fn(p(16), 4, 32, p(16), p(16), 0, p(16), 4, None) == 2
        assert fn(p(24), 4, 32, p(16), p(16), 1, p(16), 4, None) == 5
    f = lib.varlen_fold_pair_bias_row
    assert f(None, 0, 0, 1, 1, 0, 1, p(16), 1, 4, 2, None, p(16), None) == 1
    assert f(p(16), 0, 0, 1, 1, 0, 0, p(16), 1, 4, 2, None, p(16), None) == 2   # head_div 0
    assert f(p(16), 0, -1, 1, 1, 0, 1, p(16), 1, 4, 2, None, p(16), None) == 6
    assert f(p(16), 0, 0, 1, 1, 0, 1, p(16), 1, 4, 2, p(18), p(16), None) == 5


def test_decode_host_validation_codes(lib):
    p = ctypes.c_void_p

    def call(**kw):
        a = dict(q=16, cu=16, batch=2, tq=2, mq=1, kc=16, vc=16, cl=64, cs=16, kn=None, vn=None,
                 hq=8, hkv=2, d=128, scale=0.1, causal=1, splits=0, out=16, lse=16)
        a.update(kw)
        q_ = lambda x: None if x is None else p(x)
        return lib.varlen_attn_decode(q_(a["q"]), q_(a["cu"]), a["batch"], a["tq"], a["mq"],
                                      q_(a["kc"]), q_(a["vc"]), a["cl"], q_(a["cs"]), q_(a["kn"]),
                                      q_(a["vn"]), a["hq"], a["hkv"], a["d"], a["scale"],
                                      a["causal"], a["splits"], q_(a["out"]), q_(a["lse"]), None)
    assert call(q=None) == 1
    assert call(kn=16) == 1            # k_new without v_new
    assert call(batch=0) == 2
    assert call(cl=0) == 2
    assert call(splits=-1) == 2
    assert call(hq=6, hkv=4) == 3
    assert call(d=96) == 4
    assert call(mq=9, hq=8, hkv=2) == 2   # 9 x G=4 > 32 rows: the packed forward's job
    assert call(kc=24) == 5


def test_backward_host_validation_codes(lib):
    p = ctypes.c_void_p

    def call(**kw):
        a = dict(q=16, k=16, v=16, out=16, lse=16, dout=16, cuq=16, cuk=16, batch=2, tq=4, tk=4,
                 mq=2, mk=2, hq=4, hkv=2, d=64, scale=0.1, causal=1, bk=None, bp=None,
                 flags=0, dq=16, dk=16, dv=16, dbk=None, dbp=None, dsb=0)
        a.update(kw)
        q_ = lambda x: None if x is None else p(x)
        return lib.varlen_attn_bwd(
            q_(a["q"]), q_(a["k"]), q_(a["v"]), q_(a["out"]), q_(a["lse"]), q_(a["dout"]),
            q_(a["cuq"]), q_(a["cuk"]), a["batch"], a["tq"], a["tk"], a["mq"], a["mk"], a["hq"],
            a["hkv"], a["d"], a["scale"], a["causal"], q_(a["bk"]), q_(a["bp"]), 0, 0, 0, 0,
            a["flags"], q_(a["dq"]), q_(a["dk"]), q_(a["dv"]), q_(a["dbk"]), q_(a["dbp"]),
            a["dsb"], 0, 0, None)
    assert call(lse=None) == 1
    assert call(dout=None) == 1
    assert call(dk=None) == 1
    assert call(dv=None) == 1
    if not torch.cuda.is_available():       # with no keys dK/dV are never written
        assert call(k=None, v=None, dk=None, dv=None, tk=0, mk=0) == 7
    assert call(batch=0) == 2
    assert call(hq=6, hkv=4) == 3
    assert call(d=96) == 4
    assert call(dq=24) == 5
    assert call(dbp=16, dsb=-1) == 6
    assert call(flags=2) == 6
    assert call(batch=70000) == 11


def test_backward_binding_rejects_bad_tensors(lib):
    q = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    k = torch.zeros(4, 1, 64, dtype=torch.bfloat16)
    lse = torch.zeros(2, 4)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    # host tensors: the binding refuses them (no CPU path)
    with pytest.raises(ValueError):
        va.varlen_attn_bwd(q, k, k, q, lse, q, cu, cu, 4, 4)
    # wrong dtype
    with pytest.raises(ValueError):
        va.varlen_attn_bwd(q.float(), k, k, q, lse, q, cu, cu, 4, 4)
    # dout of the wrong shape
    with pytest.raises(ValueError):
        va.varlen_attn_bwd(q, k, k, q, lse, q[:2], cu, cu, 4, 4)


def test_wait_limit_setting(lib):
    # host-only: a negative limit is rejected, 0 restores the default
    assert lib.varlen_attn_set_wait_limit(-1) == 2
    assert lib.varlen_attn_set_wait_limit(1000) == 0
    assert lib.varlen_attn_set_wait_limit(0) == 0
    with pytest.raises(va.VarlenAttnError):
        va.set_wait_limit(-5)
    va.set_wait_limit(0)


def test_test_stall_setting(lib):
    assert lib.varlen_attn_set_test_stall(1) == 0
    assert lib.varlen_attn_set_test_stall(0) == 0
    va.set_test_stall(False)


def test_header_compiles_as_c99_and_links(tmp_path):
    """A plain C program (no C++, no CUDA headers) includes the header, links
    the library and calls it: the host-side argument checks answer before any
    device work, so this runs without a GPU."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use_abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "varlen_attn.h"
int main(void) {
  /* a NULL query pointer is rejected on the host */
  int rc = varlen_attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 8, 8, 8, 8, 2, 2, 64, 0.125f, 1,
                           NULL, NULL, 0, 0, 0, 0, NULL, NULL, NULL);
  if (rc != VARLEN_ATTN_ERR_NULL_POINTER) { printf("fwd rc %d\n", rc); return 1; }
  if (strlen(varlen_attn_strerror(rc)) == 0) return 2;
  if (varlen_attn_version() < 100) return 3;
  printf("ok %s\n", varlen_attn_strerror(rc));
  return 0;
}
''')
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(va.load_library()._name)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        str(src), "-L", libdir, "-lvarlen_attn", f"-Wl,-rpath,{libdir}", "-o",
                        str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")
