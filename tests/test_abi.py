"""The C-ABI library loads, exports what the header declares, and rejects bad
arguments on the host before any launch (CPU only: no compute call is made)."""
import ctypes
import os
import re

import numpy as np
import pytest

from long_context_04_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return api.lib()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(la_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for must in ("la_prefill", "la_decode_step", "la_state_out", "la_status_string",
                 "la_get_device_status"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared_functions():
        assert hasattr(L, name), name


def _declared_signatures():
    """name -> parameter kinds ("ptr", "i32", "u32", "u64") from the header declarations."""
    sigs = {}
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", fn)).read(), flags=re.S)
        for name, params in re.findall(r"\b(la_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text):
            kinds = []
            for prm in (x.strip() for x in params.split(",")):
                if prm in ("", "void"):
                    continue
                if "*" in prm:
                    kinds.append("ptr")
                elif prm.startswith("unsigned long long"):
                    kinds.append("u64")
                elif prm.startswith("unsigned"):
                    kinds.append("u32")
                elif prm.startswith(("int ", "la_status ")):
                    kinds.append("i32")
                else:
                    raise AssertionError(f"{name}: unclassified parameter {prm!r}")
            sigs[name] = kinds
    return sigs


def _ctypes_kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    return {ctypes.c_int: "i32", ctypes.c_uint: "u32", ctypes.c_ulonglong: "u64"}[t]


def test_binding_argtypes_match_the_header(L):
    """Every declared entry point is called with the header's parameter list: a drifted
    argtypes entry would pass arguments in the wrong registers without any error."""
    sigs = _declared_signatures()
    assert set(sigs) == set(_declared_functions())
    for name, kinds in sigs.items():
        got = [_ctypes_kind(t) for t in (getattr(L, name).argtypes or [])]
        assert got == kinds, (name, got, kinds)


def test_status_strings(L):
    for code, text in [(0, "LA_OK"), (1, "LA_ERR_INVALID_ARG"), (2, "LA_ERR_UNSUPPORTED"),
                       (3, "LA_ERR_CUDA"), (4, "LA_ERR_DEVICE_TIMEOUT"),
                       (5, "LA_ERR_DEVICE_RANGE")]:
        assert api.status_string(code) == text
    assert api.status_string(99) == "LA_ERR_UNKNOWN"
    assert L.la_version() >= 100


FAKE = 0x10000  # an aligned, never-dereferenced address: validation fails before any use


def _prefill(L, *, q=FAKE, o=FAKE, B=1, H=2, N=8, D=128, beta=128, cu=None, S=0, flags=1,
             st=None):
    cu_arr = None
    if cu is not None:
        arr = np.ascontiguousarray(np.asarray(cu, np.int32))
        cu_arr = arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        _prefill.keep = arr
    return L.la_prefill(q, FAKE, FAKE, o, B, H, N, D, beta, cu_arr, S, flags, st, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), api.LA_ERR_INVALID_ARG),
    (dict(o=None), api.LA_ERR_INVALID_ARG),
    (dict(q=FAKE + 2), api.LA_ERR_INVALID_ARG),          # misaligned
    (dict(H=0), api.LA_ERR_INVALID_ARG),
    (dict(N=-1), api.LA_ERR_INVALID_ARG),
    (dict(B=0), api.LA_ERR_INVALID_ARG),
    (dict(D=96), api.LA_ERR_UNSUPPORTED),
    (dict(D=256), api.LA_ERR_UNSUPPORTED),
    (dict(beta=32), api.LA_ERR_UNSUPPORTED),
    (dict(beta=256), api.LA_ERR_UNSUPPORTED),
    (dict(flags=1 | 64), api.LA_ERR_INVALID_ARG),        # unknown flag bit
    (dict(flags=1 | 4, st=None), api.LA_ERR_INVALID_ARG),  # state requested, no buffer
    (dict(flags=1 | 8, st=None), api.LA_ERR_INVALID_ARG),  # initial state, no buffer
    (dict(flags=1 | 4 | 8, st=FAKE + 4), api.LA_ERR_INVALID_ARG),  # misaligned state buffer
    (dict(flags=1 | 16), api.LA_ERR_INVALID_ARG),        # unknown flag bit
    (dict(cu=[0, 3, 8], S=2, B=2), api.LA_ERR_INVALID_ARG),  # cu_seqlens needs B == 1
    (dict(cu=[1, 3, 8], S=2), api.LA_ERR_INVALID_ARG),   # must start at 0
    (dict(cu=[0, 3, 7], S=2), api.LA_ERR_INVALID_ARG),   # must end at N
    (dict(cu=[0, 5, 3, 8], S=3), api.LA_ERR_INVALID_ARG),  # decreasing
    (dict(cu=[0], S=0), api.LA_ERR_INVALID_ARG),          # no sequence
    (dict(cu=list(range(1026)), S=1025, N=1025), api.LA_ERR_UNSUPPORTED),  # too many
])
def test_prefill_rejects(L, kw, code):
    assert _prefill(L, **kw) == code


@pytest.mark.parametrize("args,code", [
    ((None, FAKE, FAKE, FAKE, FAKE, 2, 2, 128, 1), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, None, FAKE, 2, 2, 128, 1), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE + 4, FAKE, 2, 2, 128, 1), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 128, 1), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 2, 0, 128, 1), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 2, 2, 32, 1), api.LA_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 2, 2, 128, 1 | 4), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 128, 1), api.LA_OK),   # empty batch: no-op
])
def test_decode_rejects(L, args, code):
    assert L.la_decode_step(*args, None) == code


@pytest.mark.parametrize("args,code", [
    ((None, FAKE, 2, 2, 128, None, 2), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, 3, 2, 128, None, 2), api.LA_ERR_INVALID_ARG),   # identity map overflows
    ((FAKE, FAKE, 2, 2, 100, None, 2), api.LA_ERR_UNSUPPORTED),
    ((FAKE, FAKE + 8, 2, 2, 128, None, 2), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, 0, 2, 128, None, 2), api.LA_OK),                 # nothing to copy
])
def test_state_out_rejects(L, args, code):
    assert L.la_state_out(*args, None) == code


@pytest.mark.parametrize("args,code", [
    ((FAKE, FAKE, 1, 2, 8, 128, None, 0, 1 | 2, FAKE), api.LA_ERR_INVALID_ARG),   # flag not allowed
    ((FAKE, FAKE, 1, 2, 8, 128, None, 0, 1, None), api.LA_ERR_INVALID_ARG),       # no output
    ((None, FAKE, 1, 2, 8, 128, None, 0, 1, FAKE), api.LA_ERR_INVALID_ARG),       # no k
    ((FAKE, FAKE, 1, 2, 8, 96, None, 0, 1, FAKE), api.LA_ERR_UNSUPPORTED),
    ((FAKE, FAKE, 1, 0, 8, 128, None, 0, 1, FAKE), api.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, 1, 2, 8, 128, None, 0, 1, FAKE + 8), api.LA_ERR_INVALID_ARG),   # misaligned
])
def test_chunk_state_rejects(L, args, code):
    assert L.la_chunk_state(*args, None) == code


@pytest.mark.parametrize("args,code", [
    ((FAKE, 0, 0, 1, 2, 128, FAKE), api.LA_ERR_INVALID_ARG),      # R < 1
    ((FAKE, 2, 3, 1, 2, 128, FAKE), api.LA_ERR_INVALID_ARG),      # rank > R
    ((FAKE, 2, -1, 1, 2, 128, FAKE), api.LA_ERR_INVALID_ARG),
    ((None, 2, 1, 1, 2, 128, FAKE), api.LA_ERR_INVALID_ARG),
    ((FAKE, 2, 1, 1, 2, 100, FAKE), api.LA_ERR_UNSUPPORTED),
    ((FAKE, 2, 1, 0, 2, 128, FAKE), api.LA_OK),                   # nothing to do
])
def test_state_prefix_rejects(L, args, code):
    assert L.la_state_prefix(*args, None) == code
