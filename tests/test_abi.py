"""The C-ABI boundary on CPU (no device needed, no compute calls): the
library builds for sm_100a and loads, exports every function include/msk.h
declares as a dynamic symbol, the Python binding offers the same names, and
the one host-only call (status strings) answers for every status code."""
import ctypes
import os
import re
import subprocess

import verify_step_megakernel_b200 as msk
from verify_step_megakernel_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msk.h")


def _header_text():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def declared_functions():
    return sorted(set(re.findall(r"\b(msk_[a-z0-9_]+)\s*\(", _header_text())))


def status_codes():
    return {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(MSK_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", _header_text())}


def test_header_declares_the_step_calls():
    names = declared_functions()
    for n in ("msk_create", "msk_destroy", "msk_kv_create", "msk_kv_destroy", "msk_kv_append", "msk_step",
              "msk_step_status", "msk_query", "msk_set_debug", "msk_status_string", "msk_step_static"):
        assert n in names, n


def test_library_exports_every_declared_function():
    path = _build.build()
    lib = ctypes.CDLL(path)
    names = declared_functions()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # exported as defined text symbols of the shared object itself
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.split() and line.split()[-2] in ("T", "t")}
    assert not [n for n in names if n not in syms], [n for n in names if n not in syms]


def test_binding_offers_the_same_names():
    assert sorted(msk.EXPORTS) == declared_functions()
    for n in msk.EXPORTS:
        assert callable(getattr(msk, n)), n


def test_status_strings_for_every_code():
    codes = status_codes()
    assert codes.get("MSK_OK") == 0 and len(codes) >= 8, codes
    seen = set()
    for name, v in codes.items():
        s = msk.msk_status_string(v)
        assert isinstance(s, str) and s, name
        seen.add(s)
    assert len(seen) == len(codes)  # one distinct message per code


def test_null_handles_are_refused_without_device_work():
    lib = ctypes.CDLL(_build.build())
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.msk_step.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp]
    lib.msk_step_static.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp]
    lib.msk_kv_create.argtypes = [vp, i32, i64, vp]
    lib.msk_kv_append.argtypes = [vp, vp, i32, i32, i64, i64, vp, vp, vp]
    lib.msk_kv_read.argtypes = [vp, vp, i32, i32, i64, i64, vp, vp]
    for f in ("msk_step_status", "msk_set_debug", "msk_query", "msk_destroy", "msk_kv_destroy"):
        getattr(lib, f).argtypes = [vp] if f in ("msk_step_status", "msk_destroy", "msk_kv_destroy") else [vp, vp]
    fake = 0x10000
    out = ctypes.c_void_p()
    assert lib.msk_create(None, None, 0, ctypes.byref(out)) == 1
    assert lib.msk_step(None, fake, fake, 1, 1, fake, fake, None) == 1
    assert lib.msk_step_static(None, fake, fake, 1, 1, fake, fake, None) == 1
    assert lib.msk_kv_create(None, 1, 16, ctypes.byref(out)) == 1
    assert lib.msk_kv_append(None, fake, 0, 0, 0, 1, fake, fake, None) == 1
    assert lib.msk_kv_read(None, fake, 0, 0, 0, 1, fake, fake) == 1
    assert lib.msk_step_status(None) == 1
    assert lib.msk_set_debug(None, None) == 1
    assert lib.msk_query(None, None) == 1
    lib.msk_destroy(None)     # no-ops
    lib.msk_kv_destroy(None)
