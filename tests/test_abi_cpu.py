"""CPU-only checks of the C-ABI library: it loads, exports every symbol that
include/aqua.h declares, the ctypes struct matches the C layout, and host-side
argument checks reject bad calls without touching a GPU."""
import ctypes
import os
import re

import pytest

import sparse_dimension_attention_b200 as aq
from sparse_dimension_attention_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "aqua.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"AQUA_API\s+[\w\s\*]+?\b(aqua_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    from sparse_dimension_attention_b200 import build
    build.build()
    return aq.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(abi.EXPORTED)


def test_exports_nothing_else(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True, text=True).stdout
    syms = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert syms == set(_declared())


def test_struct_layout():
    # 7 pointers followed by 8 ints on LP64
    assert ctypes.sizeof(abi.aqua_cache) == 7 * 8 + 8 * 4
    assert abi.aqua_cache.B.offset == 56
    assert abi.aqua_cache.dtype.offset == 56 + 6 * 4
    assert abi.aqua_cache.dv_store.offset == 56 + 7 * 4


def test_version(lib):
    assert aq.aqua_version() == 4


def _desc(**kw):
    base = dict(k_proj=0x1000, v=0x2000, len=0x3000, n_abs=0x3100, pos=None, score=None, ctrl=0x4000,
                B=2, Hkv=2, d=128, d_store=128, Tcap=64, max_len=0, dtype=abi.AQUA_BF16)
    base.update(kw)
    return abi.aqua_cache(**base)


@pytest.mark.parametrize("field,value,code", [
    ("d", 64, abi.AQUA_ERR_UNSUPPORTED),
    ("d_store", 0, abi.AQUA_ERR_ARG),
    ("d_store", 129, abi.AQUA_ERR_ARG),
    ("Tcap", 40, abi.AQUA_ERR_ARG),
    ("dtype", 7, abi.AQUA_ERR_UNSUPPORTED),
    ("k_proj", None, abi.AQUA_ERR_ARG),
    ("k_proj", 0x1004, abi.AQUA_ERR_ARG),       # misaligned
    ("max_len", 65, abi.AQUA_ERR_ARG),
    ("dv_store", 8, abi.AQUA_ERR_ARG),         # not a multiple of 16
    ("dv_store", 144, abi.AQUA_ERR_ARG),
    ("dv_store", -16, abi.AQUA_ERR_ARG),
])
def test_project_keys_rejects_bad_cache(lib, field, value, code):
    c = _desc(**{field: value})
    rc = lib.aqua_project_keys(ctypes.byref(c), 0x5000, 0x6000, 0x7000, 1, None)
    assert rc == code
    assert lib.aqua_last_error().decode() != ""


def test_project_keys_rejects_overflow(lib):
    c = _desc(max_len=60)
    assert lib.aqua_project_keys(ctypes.byref(c), 0x5000, 0x6000, 0x7000, 5, None) == abi.AQUA_ERR_ARG
    assert c.max_len == 60     # unchanged on failure
    assert lib.aqua_project_keys(ctypes.byref(c), 0x5000, 0x6000, 0x7000, 0, None) == abi.AQUA_ERR_ARG


def test_decode_argument_checks(lib):
    c = _desc()
    ws = lib.aqua_decode_workspace_size(ctypes.byref(c), 8)
    assert ws > 0
    call = lambda **kw: lib.aqua_decode_attn(
        ctypes.byref(kw.get("c", c)), kw.get("q", 0x5000), kw.get("kn", None), kw.get("vn", None), 0x7000,
        kw.get("Hq", 8), kw.get("k", 96), 0.0, 0x8000, kw.get("od", abi.AQUA_BF16), None, None, None, None,
        kw.get("ws", 0x10000), kw.get("wsb", ws), None)
    assert call(Hq=7) == abi.AQUA_ERR_ARG                 # not a multiple of Hkv
    assert call(Hq=16) == abi.AQUA_ERR_UNSUPPORTED        # group of 8
    assert call(k=0) == abi.AQUA_ERR_ARG
    assert call(k=129) == abi.AQUA_ERR_ARG
    assert call(c=_desc(d_store=96), k=97) == abi.AQUA_ERR_ARG
    assert call(q=None) == abi.AQUA_ERR_ARG
    assert call(od=5) == abi.AQUA_ERR_UNSUPPORTED
    assert call(wsb=ws - 1) == abi.AQUA_ERR_WORKSPACE
    assert call(ws=0x10010) == abi.AQUA_ERR_ARG           # workspace alignment
    assert call(kn=0x9000) == abi.AQUA_ERR_ARG            # k_new without v_new
    full = _desc(max_len=64)
    assert call(c=full, kn=0x9000, vn=0x9100) == abi.AQUA_ERR_ARG   # no room to append
    assert full.max_len == 64


def test_decode_phases_argument_checks(lib):
    """aqua_decode_select / aqua_decode_attend check the arguments each one uses."""
    c = _desc(max_len=10)
    ws = lib.aqua_decode_workspace_size(ctypes.byref(c), 8)
    sel = lambda **kw: lib.aqua_decode_select(
        ctypes.byref(kw.get("c", c)), kw.get("q", 0x5000), kw.get("kn", None), kw.get("vn", None), 0x7000,
        kw.get("Hq", 8), kw.get("k", 96), 0.0, None, None, kw.get("ws", 0x10000), kw.get("wsb", ws), None)
    att = lambda **kw: lib.aqua_decode_attend(
        ctypes.byref(kw.get("c", c)), kw.get("P", None), kw.get("Hq", 8), kw.get("app", 0), kw.get("out", 0x8000),
        kw.get("od", abi.AQUA_BF16), None, None, kw.get("ws", 0x10000), kw.get("wsb", ws), None)
    assert sel(q=None) == abi.AQUA_ERR_ARG
    assert sel(k=0) == abi.AQUA_ERR_ARG
    assert sel(Hq=16) == abi.AQUA_ERR_UNSUPPORTED
    assert sel(kn=0x9000) == abi.AQUA_ERR_ARG
    assert sel(wsb=ws - 1) == abi.AQUA_ERR_WORKSPACE
    assert att(app=2) == abi.AQUA_ERR_ARG
    assert att(c=_desc(max_len=0), app=1) == abi.AQUA_ERR_ARG       # nothing was appended
    assert att(out=None) == abi.AQUA_ERR_ARG
    assert att(od=9) == abi.AQUA_ERR_UNSUPPORTED
    assert att(Hq=7) == abi.AQUA_ERR_ARG
    assert att(ws=0x10010) == abi.AQUA_ERR_ARG
    cv = _desc(max_len=10, dv_store=96)
    wsv = lib.aqua_decode_workspace_size(ctypes.byref(cv), 8)
    assert wsv > ws                                                   # room for the pre-projection outputs
    assert att(c=cv, wsb=wsv) == abi.AQUA_ERR_ARG                     # projected values need P
    assert att(c=cv, P=0x7004, wsb=wsv) == abi.AQUA_ERR_ARG          # misaligned P
    assert att(c=cv, wsb=ws, P=0x7000) == abi.AQUA_ERR_WORKSPACE
    assert c.max_len == 10


def test_static_decode_checks_match_the_workspace_entry_point(lib):
    """aqua_decode_attn_static rejects bad calls with aqua_decode_attn's codes,
    before it compares the shape's scratch with its built-in array."""
    def both(c, Hq, k=96, od=abi.AQUA_BF16, q=0x5000):
        ws_call = lib.aqua_decode_attn(ctypes.byref(c), q, None, None, 0x7000, Hq, k, 0.0, 0x8000, od, None, None,
                                       None, None, 0x10000, 1 << 40, None)
        st_call = lib.aqua_decode_attn_static(ctypes.byref(c), q, None, None, 0x7000, Hq, k, 0.0, 0x8000, od, None,
                                              None, None, None, None)
        return ws_call, st_call
    big = _desc(B=512, Hkv=8)
    assert both(big, 64) == (abi.AQUA_ERR_UNSUPPORTED, abi.AQUA_ERR_UNSUPPORTED)   # group of 8, not scratch
    assert both(big, 12) == (abi.AQUA_ERR_ARG, abi.AQUA_ERR_ARG)
    assert both(big, 32, k=0) == (abi.AQUA_ERR_ARG, abi.AQUA_ERR_ARG)
    assert both(big, 32, od=4) == (abi.AQUA_ERR_UNSUPPORTED, abi.AQUA_ERR_UNSUPPORTED)
    assert both(_desc(d=64), 8) == (abi.AQUA_ERR_UNSUPPORTED, abi.AQUA_ERR_UNSUPPORTED)
    assert both(big, 32, q=None) == (abi.AQUA_ERR_ARG, abi.AQUA_ERR_ARG)
    # a valid call whose scratch exceeds the 8 MiB array
    st = lib.aqua_decode_attn_static(ctypes.byref(big), 0x5000, None, None, 0x7000, 32, 96, 0.0, 0x8000,
                                     abi.AQUA_BF16, None, None, None, None, None)
    assert st == abi.AQUA_ERR_WORKSPACE
    assert "8388608" in lib.aqua_last_error().decode()


def test_decode_workspace_grows_with_units(lib):
    a = lib.aqua_decode_workspace_size(ctypes.byref(_desc(B=1, Hkv=1)), 4)
    b = lib.aqua_decode_workspace_size(ctypes.byref(_desc(B=8, Hkv=8)), 32)
    assert 0 < a < b
    assert lib.aqua_decode_workspace_size(ctypes.byref(_desc()), 3) == 0


def test_h2o_argument_checks(lib):
    c = _desc()
    assert lib.aqua_h2o_update(ctypes.byref(c), 0x5000, 0x6000, 8, 16, 4, None, None) == abi.AQUA_ERR_ARG  # no pos
    c = _desc(pos=0x9000, score=0x9100)
    assert lib.aqua_h2o_update(ctypes.byref(c), 0x5000, 0x6000, 8, 16, 17, None, None) == abi.AQUA_ERR_ARG
    assert lib.aqua_h2o_update(ctypes.byref(c), 0x5000, 0x6000, 8, 0, 0, None, None) == abi.AQUA_ERR_ARG
    # group sizes the decode step does not produce: rejected before any launch
    assert lib.aqua_h2o_update(ctypes.byref(c), 0x5000, 0x6000, 3 * c.Hkv, 16, 4, None, None) == \
        abi.AQUA_ERR_UNSUPPORTED


def test_selftest_argument_checks(lib):
    c = _desc()
    assert lib.aqua_selftest_wait_timeout(ctypes.byref(c), 10, None) == abi.AQUA_ERR_ARG        # under 1 us
    assert lib.aqua_selftest_wait_timeout(ctypes.byref(c), 3 * 10 ** 9, None) == abi.AQUA_ERR_ARG  # over 2 s
    nc = _desc(ctrl=None)
    assert lib.aqua_selftest_wait_timeout(ctypes.byref(nc), 10 ** 6, None) == abi.AQUA_ERR_ARG


def test_prefill_argument_checks(lib):
    c = _desc()
    ws = lib.aqua_prefill_workspace_size(ctypes.byref(c), 8, 32)
    assert lib.aqua_prefill_attn(ctypes.byref(c), 0x5000, 40, 32, 0x7000, 8, 96, 0.0, 0x8000, abi.AQUA_BF16,
                                 None, None, 0x10000, ws, None) == abi.AQUA_ERR_ARG   # pos0 + L > Tcap
    cv = _desc(dv_store=64)
    assert lib.aqua_prefill_attn(ctypes.byref(cv), 0x5000, 0, 32, 0x7000, 8, 96, 0.0, 0x8000, abi.AQUA_BF16,
                                 None, None, 0x10000, ws, None) == abi.AQUA_ERR_UNSUPPORTED   # decode-only
    c32 = _desc(dtype=abi.AQUA_F32)
    assert lib.aqua_prefill_attn(ctypes.byref(c32), 0x5000, 0, 32, 0x7000, 8, 96, 0.0, 0x8000, abi.AQUA_BF16,
                                 None, None, 0x10000, ws, None) == abi.AQUA_ERR_UNSUPPORTED
    assert lib.aqua_prefill_attn(ctypes.byref(c), 0x5000, 0, 32, 0x7000, 8, 96, 0.0, 0x8000, abi.AQUA_BF16,
                                 None, 0x9004, 0x10000, ws, None) == abi.AQUA_ERR_ARG  # qproj_out misaligned


def test_calibrate_argument_checks(lib):
    assert lib.aqua_calibrate_workspace_size(16384, 128) > 0
    assert lib.aqua_calibrate_workspace_size(16384, 64) == 0
    assert lib.aqua_calibrate(0x1000, 10, 64, 0x2000, 0x3000, 0x4000, 1 << 30, None) == abi.AQUA_ERR_UNSUPPORTED
    need = lib.aqua_calibrate_workspace_size(100, 128)
    assert lib.aqua_calibrate(0x1000, 100, 128, 0x2000, 0x3000, 0x4000, need - 8, None) == abi.AQUA_ERR_WORKSPACE


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "sparse_dimension_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "aqua_oracle" not in txt, f


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(abi, "_lib", None)
    with pytest.raises(RuntimeError):
        abi.load_library(str(tmp_path / "nope.so"))
