"""The C-ABI library: it loads, exports every function include/pw.h declares, and its
host-only logic (sizes, argument checks) is right.  No call here reaches a GPU."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from dynamic_sparse_attention_pw_b200 import _lib, api, build
from dynamic_sparse_attention_pw_b200 import synth
from oracle import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.load()


def _declared_functions():
    names = []
    for hdr in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not hdr.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(pw_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_function_is_exported(L):
    declared = _declared_functions()
    assert set(declared) >= {"pw_groups_size", "pw_group", "pw_attn"}
    for name in declared:
        assert hasattr(L, name), name
    assert set(_lib.EXPORTED) <= set(declared)


def test_version_and_status_strings(L):
    assert L.pw_version() >= 100
    for code in range(7):
        assert len(_lib.status_string(code)) > 0


def _sizes(L, cu, Hkv, kmax, W, g):
    cu = np.ascontiguousarray(cu, np.int32)
    ng, uc, wd, ws = C.c_int64(), C.c_int64(), C.c_int32(), C.c_size_t()
    st = L.pw_groups_size(cu.ctypes.data_as(C.c_void_p), len(cu) - 1, Hkv, kmax, W, g,
                          C.byref(ng), C.byref(uc), C.byref(wd), C.byref(ws))
    return st, ng.value, uc.value, wd.value, ws.value


@pytest.mark.parametrize("seqlens,Hkv,kmax,W,g", [
    ((1024,), 1, 4, 32, 8),
    ((8192, 16384, 32768, 65536), 8, 64, 128, 8),
    ((70, 129, 300, 1), 2, 5, 24, 3),
    ((0, 64, 0, 65), 3, 7, 8, 8),
    ((131072,), 1, 2, 256, 32),
])
def test_groups_size_matches_oracle_counts(L, seqlens, Hkv, kmax, W, g):
    cu = synth.cu_seqlens_of(seqlens)
    st, ng, uc, words, ws = _sizes(L, cu, Hkv, kmax, W, g)
    assert st == _lib.PW_OK
    ong, oucap = oracle.group_counts(cu, Hkv, kmax, W, g)
    assert ng == ong and uc == oucap
    maxp = max((n + 63) // 64 for n in seqlens)
    assert words == max(1, (maxp + 31) // 32)
    assert ws >= 256 and ws % 256 == 0


@pytest.mark.parametrize("W,g,code", [
    (30, 8, _lib.PW_ERR_UNSUPPORTED),   # W not a multiple of g
    (512, 8, _lib.PW_ERR_UNSUPPORTED),  # W above 256
    (64, 33, _lib.PW_ERR_UNSUPPORTED),  # g above 32
    (0, 8, _lib.PW_ERR_INVALID_ARG),
    (8, 0, _lib.PW_ERR_INVALID_ARG),
])
def test_groups_size_rejects_unsupported(L, W, g, code):
    st, *_ = _sizes(L, [0, 100], 1, 4, W, g)
    assert st == code


def test_groups_size_rejects_bad_offsets_and_long_sequences(L):
    assert _sizes(L, [5, 100], 1, 4, 8, 8)[0] == _lib.PW_ERR_INVALID_ARG
    assert _sizes(L, [0, 100, 50], 1, 4, 8, 8)[0] == _lib.PW_ERR_INVALID_ARG
    assert _sizes(L, [0, 131072 + 64], 1, 4, 8, 8)[0] == _lib.PW_ERR_UNSUPPORTED


def test_calls_reject_bad_arguments_before_any_device_work(L):
    cu = np.array([0, 128], np.int32)
    cup = cu.ctypes.data_as(C.c_void_p)
    g = _lib.PwGroups()
    # no groups struct
    st = L.pw_group(C.c_void_p(16), C.c_void_p(16), cup, 1, 1, 4, 32, 8, None, C.c_void_p(256),
                    1 << 20, C.c_void_p(16), None)
    assert st == _lib.PW_ERR_INVALID_ARG
    # struct that does not match the sizes
    g.g, g.words, g.n_groups = 8, 1, 999
    st = L.pw_group(C.c_void_p(16), C.c_void_p(16), cup, 1, 1, 4, 32, 8, C.byref(g),
                    C.c_void_p(256), 1 << 20, C.c_void_p(16), None)
    assert st == _lib.PW_ERR_INVALID_ARG
    # too small a workspace
    g.n_groups = 16
    g.union_cap = 16 * 2
    st = L.pw_group(C.c_void_p(16), C.c_void_p(16), cup, 1, 1, 4, 32, 8, C.byref(g),
                    C.c_void_p(256), 0, C.c_void_p(16), None)
    assert st == _lib.PW_ERR_CAPACITY
    # attention: tile rows above 128, misaligned pointers, missing groups
    g.g = 32
    st = L.pw_attn(C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), 2, 2,
                   C.c_void_p(16), 1, 128, 16, 2, 1.0, 1.0, 0.1, C.byref(g), C.c_void_p(16),
                   C.c_void_p(16), None)
    assert st == _lib.PW_ERR_UNSUPPORTED
    g.g = 8
    st = L.pw_attn(C.c_void_p(17), C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), 2, 2,
                   C.c_void_p(16), 1, 128, 16, 2, 1.0, 1.0, 0.1, C.byref(g), C.c_void_p(16),
                   C.c_void_p(16), None)
    assert st == _lib.PW_ERR_INVALID_ARG
    st = L.pw_attn(C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), 2, 2,
                   C.c_void_p(16), 1, 128, 16, 3, 1.0, 1.0, 0.1, C.byref(g), C.c_void_p(16),
                   C.c_void_p(16), None)
    assert st == _lib.PW_ERR_UNSUPPORTED   # Hq not a multiple of Hkv
    st = L.pw_attn(C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), 2, 2,
                   C.c_void_p(16), 1, 128, 16, 2, 1.0, 1.0, 0.1, None, C.c_void_p(16),
                   C.c_void_p(16), None)
    assert st == _lib.PW_ERR_INVALID_ARG
    # groups whose arrays are all given except the work counter
    for f in ("qids", "gsize", "gmeta", "union_off", "union_pages", "bits"):
        setattr(g, f, 256)
    g.sched = None
    st = L.pw_attn(C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), 2, 2,
                   C.c_void_p(16), 1, 128, 16, 2, 1.0, 1.0, 0.1, C.byref(g), C.c_void_p(16),
                   C.c_void_p(16), None)
    assert st == _lib.PW_ERR_INVALID_ARG


def test_device_status_codes_reach_the_caller_by_name():
    """What a kernel records in the status word (a bounded wait that ran out, a bad selection,
    an out-of-range page-table entry) is raised by check_status with the code's name."""
    import torch
    for code, word in ((_lib.PW_ERR_TIMEOUT, "wait"), (_lib.PW_ERR_BAD_SELECTION, "selected"),
                       (_lib.PW_ERR_INVALID_ARG, "")):
        with pytest.raises(_lib.PwError) as e:
            api.check_status(torch.tensor([code], dtype=torch.int32), "test")
        assert word in str(e.value).lower()
    api.check_status(torch.zeros(1, dtype=torch.int32), "test")


def test_product_path_has_no_fallback():
    # The binding must raise, not compute elsewhere, when the library is absent.
    import importlib
    saved = _lib.LIB_PATH, _lib._lib
    try:
        _lib._lib = None
        _lib.LIB_PATH = os.path.join(ROOT, "does-not-exist", "libpw.so")
        with pytest.raises(RuntimeError):
            _lib.load()
    finally:
        _lib.LIB_PATH, _lib._lib = saved
    pkg = os.path.join(ROOT, "dynamic_sparse_attention_pw_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert not re.search(r"^\s*(import|from)\s+oracle\b", src, flags=re.M), fn
