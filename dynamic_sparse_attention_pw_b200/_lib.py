"""ctypes loader of libpw.so (the C ABI declared in include/pw.h).

No fallback: if the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpw.so")

PW_OK, PW_ERR_INVALID_ARG, PW_ERR_UNSUPPORTED, PW_ERR_BAD_SELECTION, PW_ERR_CAPACITY, \
    PW_ERR_TIMEOUT, PW_ERR_CUDA = range(7)

EXPORTED = ("pw_version", "pw_status_string", "pw_groups_size", "pw_group", "pw_attn")


class PwGroups(C.Structure):
    """Mirror of struct pw_groups."""
    _fields_ = [
        ("qids", C.c_void_p),
        ("gsize", C.c_void_p),
        ("gmeta", C.c_void_p),
        ("union_off", C.c_void_p),
        ("union_pages", C.c_void_p),
        ("bits", C.c_void_p),
        ("sched", C.c_void_p),
        ("n_groups", C.c_int64),
        ("union_cap", C.c_int64),
        ("words", C.c_int32),
        ("g", C.c_int32),
    ]


class PwError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


_lib = None


def load() -> C.CDLL:
    """Load libpw.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m dynamic_sparse_attention_pw_b200.build`")
    L = C.CDLL(LIB_PATH)
    p, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
    L.pw_version.argtypes = []
    L.pw_version.restype = C.c_int
    L.pw_status_string.argtypes = [C.c_int]
    L.pw_status_string.restype = C.c_char_p
    L.pw_groups_size.argtypes = [p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                 C.POINTER(i64), C.POINTER(i64), C.POINTER(i32), C.POINTER(sz)]
    L.pw_groups_size.restype = C.c_int
    L.pw_group.argtypes = [p, p, p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                           C.POINTER(PwGroups), p, sz, p, p]
    L.pw_group.restype = C.c_int
    L.pw_attn.argtypes = [p, p, p, p, C.c_int, C.c_int, p, C.c_int, i64, C.c_int, C.c_int,
                          f32, f32, f32, C.POINTER(PwGroups), p, p, p]
    L.pw_attn.restype = C.c_int
    _lib = L
    return L


def status_string(code: int) -> str:
    return load().pw_status_string(int(code)).decode()
