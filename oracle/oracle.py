"""ctypes binding of the plain-C fp64 oracle (pw_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the CPU-baseline
legs of bench.py.  The product path never imports this module.  It shares no code with the
CUDA library; the only thing both sides share is the seeded input generator.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pw_oracle.c")
LIB = os.path.join(HERE, "libpw_oracle.so")
PAGE = 64
D = 128

_lib = None


def build(force: bool = False) -> str:
    """Compile pw_oracle.c into libpw_oracle.so (plain C, -O2, OpenMP)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wno-unknown-pragmas",
               "-o", LIB, SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        p = C.c_void_p
        i32, i64, f64 = C.c_int32, C.c_int64, C.c_double
        L.pwo_e4m3_to_double.argtypes = [C.c_uint8]
        L.pwo_e4m3_to_double.restype = f64
        L.pwo_bf16_to_double.argtypes = [C.c_uint16]
        L.pwo_bf16_to_double.restype = f64
        L.pwo_double_to_bf16.argtypes = [f64]
        L.pwo_double_to_bf16.restype = C.c_uint16
        L.pwo_validate.argtypes = [p, p, C.c_int, C.c_int, C.c_int]
        L.pwo_validate.restype = C.c_int
        L.pwo_group.argtypes = [p, p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, i64, i64,
                                p, p, p, p, p, p, p]
        L.pwo_group.restype = C.c_int
        L.pwo_attn_rows.argtypes = [p, p, p, p, C.c_int, p, C.c_int, C.c_int, C.c_int, C.c_int, p,
                                    f64, f64, f64, p, p, i64, C.c_int, p]
        L.pwo_attn_rows.restype = C.c_int
        L.pwo_attn_grouped.argtypes = [p, p, p, p, C.c_int, p, C.c_int, C.c_int, C.c_int, C.c_int,
                                       p, f64, f64, f64, p, p, p, p, p, i64, C.c_int, C.c_int, p]
        L.pwo_attn_grouped.restype = C.c_int
        L.pwo_double_to_bf16_n.argtypes = [p, p, i64]
        L.pwo_double_to_bf16_n.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- number formats ------------------------------------------------------------------------

def e4m3_to_f64(codes) -> np.ndarray:
    L = lib()
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([L.pwo_e4m3_to_double(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def bf16_to_f64(bits) -> np.ndarray:
    L = lib()
    bits = np.asarray(bits, dtype=np.uint16)
    flat = np.array([L.pwo_bf16_to_double(int(b)) for b in bits.ravel()], dtype=np.float64)
    return flat.reshape(bits.shape)


def f64_to_bf16(x) -> np.ndarray:
    """binary64 -> bf16 bits, round to nearest even (elementwise through the C routine)."""
    L = lib()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    L.pwo_double_to_bf16_n(_ptr(x), _ptr(out), x.size)
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bits -> binary64 values (exact), vectorised through a 65536-entry table."""
    global _BF16_TABLE
    if _BF16_TABLE is None:
        _BF16_TABLE = bf16_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    return _BF16_TABLE[np.asarray(bits, dtype=np.uint16)]


_BF16_TABLE = None


# ---- grouping ------------------------------------------------------------------------------

def group_counts(cu, Hkv: int, kmax: int, W: int, g: int):
    """(number of groups, an upper bound on the total union length) for the fixed-window
    partition: every window of n tokens yields ceil(n / g) groups."""
    cu = np.asarray(cu, dtype=np.int64)
    ng = 0
    ucap = 0
    for b in range(len(cu) - 1):
        n = int(cu[b + 1] - cu[b])
        P = (n + PAGE - 1) // PAGE
        gb = 0
        for lo in range(0, n, W):
            m = min(W, n - lo)
            gb += (m + g - 1) // g
        ng += gb * Hkv
        ucap += gb * Hkv * min(g * kmax, P)
    return ng, ucap


def group(sel, cu, W: int, g: int, with_order: bool = False) -> dict:
    """Run the oracle greedy; returns numpy arrays sized to the actual group count."""
    L = lib()
    sel = _c(sel, np.int32)
    cu = _c(cu, np.int32)
    T, Hkv, kmax = sel.shape
    B = len(cu) - 1
    cap, ucap = group_counts(cu, Hkv, kmax, W, g)
    qids = np.full(max(cap, 1) * g, -1, np.int32)
    gsize = np.zeros(max(cap, 1), np.int32)
    gmeta = np.zeros(max(cap, 1) * 3, np.int32)
    uoff = np.zeros(cap + 1, np.int32)
    upages = np.zeros(max(ucap, 1), np.int32)
    order = np.full(max(cap, 1) * g, -1, np.int32) if with_order else None
    ng = C.c_int64(0)
    st = L.pwo_group(_ptr(sel), _ptr(cu), B, Hkv, kmax, W, g, cap, ucap, _ptr(qids), _ptr(gsize),
                     _ptr(gmeta), _ptr(uoff), _ptr(upages),
                     _ptr(order) if with_order else None, C.byref(ng))
    n = ng.value
    out = {
        "status": st,
        "n_groups": n,
        "qids": qids[: n * g].reshape(n, g),
        "gsize": gsize[:n],
        "gmeta": gmeta[: 3 * n].reshape(n, 3),
        "union_off": uoff[: n + 1],
        "union_pages": upages[: int(uoff[n]) if n > 0 else 0],
        "g": g,
    }
    if with_order:
        out["order"] = order[: n * g].reshape(n, g)
    return out


def validate(sel, cu) -> int:
    sel = _c(sel, np.int32)
    cu = _c(cu, np.int32)
    T, Hkv, kmax = sel.shape
    return lib().pwo_validate(_ptr(sel), _ptr(cu), len(cu) - 1, Hkv, kmax)


# ---- attention -----------------------------------------------------------------------------

def _attn_common(inp):
    Q = _c(inp["Q"], np.uint16)
    K = _c(inp["K_pages"], np.uint8)
    V = _c(inp["V_pages"], np.uint8)
    pt = _c(inp["page_table"], np.int32)
    cu = _c(inp["cu_seqlens"], np.int32)
    sel = _c(inp["sel_pages"], np.int32)
    T, Hq, _ = Q.shape
    _, Hkv, kmax = sel.shape
    return Q, K, V, pt, cu, sel, T, Hq, Hkv, kmax


def attn_rows(inp: dict, rows_t, rows_hq, nthreads: int = 0) -> np.ndarray:
    """O (binary64) [n, 128] for the listed (token, query-head) rows, by definition."""
    L = lib()
    Q, K, V, pt, cu, sel, T, Hq, Hkv, kmax = _attn_common(inp)
    rt = _c(rows_t, np.int64)
    rh = _c(rows_hq, np.int32)
    O = np.zeros((len(rt), D), np.float64)
    nthreads = nthreads or os.cpu_count() or 1
    st = L.pwo_attn_rows(_ptr(Q), _ptr(K), _ptr(V), _ptr(pt), pt.shape[1], _ptr(cu), len(cu) - 1,
                         Hq, Hkv, kmax, _ptr(sel), float(inp["k_scale"]), float(inp["v_scale"]),
                         float(inp["sm_scale"]), _ptr(rt), _ptr(rh), len(rt), nthreads, _ptr(O))
    if st != 0:
        raise ValueError(f"oracle attn_rows status {st}")
    return O


def attn_all(inp: dict, nthreads: int = 0) -> np.ndarray:
    """O (binary64) [T, Hq, 128] for every row."""
    Q = inp["Q"]
    T, Hq, _ = Q.shape
    rt = np.repeat(np.arange(T, dtype=np.int64), Hq)
    rh = np.tile(np.arange(Hq, dtype=np.int32), T)
    return attn_rows(inp, rt, rh, nthreads).reshape(T, Hq, D)


def attn_grouped(inp: dict, groups: dict, nthreads: int = 0) -> np.ndarray:
    """O (binary64) [T, Hq, 128] reached by walking each group's union with membership masks."""
    L = lib()
    Q, K, V, pt, cu, sel, T, Hq, Hkv, kmax = _attn_common(inp)
    O = np.zeros((T, Hq, D), np.float64)
    qids = _c(groups["qids"], np.int32)
    gsize = _c(groups["gsize"], np.int32)
    gmeta = _c(groups["gmeta"], np.int32)
    uoff = _c(groups["union_off"], np.int32)
    upag = _c(groups["union_pages"], np.int32)
    if upag.size == 0:
        upag = np.zeros(1, np.int32)
    nthreads = nthreads or os.cpu_count() or 1
    st = L.pwo_attn_grouped(_ptr(Q), _ptr(K), _ptr(V), _ptr(pt), pt.shape[1], _ptr(cu), len(cu) - 1,
                            Hq, Hkv, kmax, _ptr(sel), float(inp["k_scale"]), float(inp["v_scale"]),
                            float(inp["sm_scale"]), _ptr(qids), _ptr(gsize), _ptr(gmeta), _ptr(uoff),
                            _ptr(upag), int(groups["n_groups"]), int(groups["g"]), nthreads, _ptr(O))
    if st != 0:
        raise ValueError(f"oracle attn_grouped status {st}")
    return O
