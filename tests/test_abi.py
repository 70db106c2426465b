"""Host-side checks of the C ABI: the library builds, loads and exports every
entry point include/zo.h declares; argument errors are reported without a GPU."""
import ctypes
import glob
import os
import re

import pytest

import zero_order_recurrent_b200 as zo
from zero_order_recurrent_b200 import build as zbuild

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


@pytest.fixture(scope="module")
def lib():
    zbuild.build()
    return zo.load_library()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(INCLUDE, "*.h")):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\bZO_API\s+[^;(]*?\b(zo_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(zo.EXPORTS)


def test_header_constants_match_the_binding():
    src = "".join(open(h).read() for h in glob.glob(os.path.join(INCLUDE, "*.h")))
    defines = dict(re.findall(r"#define\s+(ZO_[A-Z0-9_]+)\s+(-?\d+)\b", src))
    assert defines, "no integer constants found in the headers"
    for name, value in defines.items():
        assert getattr(zo, name) == int(value), name


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_only_declared_symbols_are_exported(lib):
    out = os.popen(f"nm -D --defined-only {zo.LIB_PATH}").read()
    syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert {s for s in syms if s.startswith("zo_")} == set(declared_functions())


def test_status_strings(lib):
    for st in range(9):
        assert zo.status_string(st)
    assert zo.status_string(ZO := zo.ZO_ERR_BOUNDS) == "token or target out of range"


def test_argument_errors_need_no_device(lib):
    h = ctypes.c_void_p()
    assert lib.zo_create(None, ctypes.byref(h)) == zo.ZO_ERR_INVALID_ARG
    bad = zo.ModelSpec(1, 4, 4, 1, 0, 1, 1, 0)          # vocab < 2
    assert lib.zo_create(ctypes.byref(bad), ctypes.byref(h)) == zo.ZO_ERR_INVALID_ARG
    bad = zo.ModelSpec(10, 4, 4, 9, 0, 1, 1, 0)         # too many layers
    assert lib.zo_create(ctypes.byref(bad), ctypes.byref(h)) == zo.ZO_ERR_INVALID_ARG
    bad = zo.ModelSpec(10, 4, 4, 1, 7, 1, 1, 0)         # unknown dtype
    assert lib.zo_create(ctypes.byref(bad), ctypes.byref(h)) == zo.ZO_ERR_INVALID_ARG
    assert lib.zo_probe_losses(None, None, 0, 1, 1e-3, None, None, 1, 1, None, None, None) == \
        zo.ZO_ERR_INVALID_ARG
    assert lib.zo_update(None, None, 0, 1, None, None) == zo.ZO_ERR_INVALID_ARG
    assert lib.zo_loss(None, None, None, None, 1, 1, None, None) == zo.ZO_ERR_INVALID_ARG
    assert lib.zo_coeffs_forward(None, None, None, 1, 1e-3, 1e-3, None, None) == \
        zo.ZO_ERR_INVALID_ARG
    assert lib.zo_sign_words(0, -1, 0, 1, None, None) == zo.ZO_ERR_INVALID_ARG


def test_create_without_device_reports_no_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    spec = zo.ModelSpec(10, 16, 32, 1, 0, 8, 21, 0)
    assert lib.zo_create(ctypes.byref(spec), ctypes.byref(h)) == zo.ZO_ERR_NO_DEVICE
    assert not h.value
