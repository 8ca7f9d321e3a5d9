"""Pins of the oracle's per-query attention.

Each query attends to exactly the keys of its own selected pages, up to its own position,
and owns its whole output ("PageWeaver: KV-Guided Query Unions for Sparse Attention",
Abstract: original support and complete output ownership are preserved).  That is plain
masked softmax attention, so the oracle is checked against a dense masked softmax written
with numpy matrix operations (decoding FP8 through ml_dtypes, not through the oracle), against
closed forms, and against the invariances the method promises.
"""
from fractions import Fraction
import math

import ml_dtypes
import numpy as np
import pytest

from dynamic_sparse_attention_pw_b200 import synth
from oracle import oracle

PAGE, D = 64, 128


def _wl(seed, seqlens, Hq, Hkv, kmax, selection="uniform", **kw):
    return synth.Workload(f"attn{seed}", 200 + seed, tuple(seqlens), Hq=Hq, Hkv=Hkv, kmax=kmax,
                          selection=selection, **kw)


def dense_masked_attention(inp):
    """Brute force: for each sequence and head, dense scores over all keys of the sequence,
    mask = (key page selected by the query) and (key position <= query position)."""
    Q = inp["Q"].view(ml_dtypes.bfloat16).astype(np.float64)
    K = inp["K_pages"].view(ml_dtypes.float8_e4m3fn).astype(np.float64) * inp["k_scale"]
    V = inp["V_pages"].view(ml_dtypes.float8_e4m3fn).astype(np.float64) * inp["v_scale"]
    sel, cu, pt = inp["sel_pages"], inp["cu_seqlens"], inp["page_table"]
    T, Hq, _ = Q.shape
    Hkv = sel.shape[1]
    G = Hq // Hkv
    O = np.zeros((T, Hq, D))
    for b in range(len(cu) - 1):
        s, e = cu[b], cu[b + 1]
        n = e - s
        if n == 0:
            continue
        pos = np.arange(n)
        phys = pt[b, pos // PAGE]
        for h in range(Hkv):
            Kd = K[phys, h, pos % PAGE]          # [n, D]
            Vd = V[phys, h, pos % PAGE]
            member = np.zeros((n, n), bool)
            for i in range(n):
                pages = sel[s + i, h]
                member[i] = np.isin(pos // PAGE, pages[pages >= 0])
            mask = member & (pos[None, :] <= pos[:, None])
            for j in range(G):
                hq = h * G + j
                S = (Q[s:e, hq] @ Kd.T) * inp["sm_scale"]
                S = np.where(mask, S, -np.inf)
                m = S.max(axis=1, keepdims=True)
                m = np.where(np.isfinite(m), m, 0.0)
                P = np.exp(S - m)
                l = P.sum(axis=1, keepdims=True)
                O[s:e, hq] = np.where(l > 0, (P @ Vd) / np.where(l > 0, l, 1), 0.0)
    return O


@pytest.mark.parametrize("wl", [
    _wl(1, [200, 64, 1, 130], Hq=6, Hkv=2, kmax=5, shuffled_pages=True),
    _wl(2, [256], Hq=8, Hkv=1, kmax=4, selection="fixed2"),
    _wl(3, [512, 96], Hq=4, Hkv=2, kmax=6, selection="community", communities=3),
])
def test_oracle_equals_dense_masked_softmax(wl):
    inp = synth.make_inputs(wl)
    ours = oracle.attn_all(inp)
    ref = dense_masked_attention(inp)
    assert np.max(np.abs(ours - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_oracle_equals_dense_on_first_benchmark_workload():
    wl = synth.WORKLOADS[1]
    inp = synth.make_inputs(wl)
    ours = oracle.attn_all(inp)
    ref = dense_masked_attention(inp)
    assert np.max(np.abs(ours - ref)) <= 1e-12


def _constant_codes(shape, code):
    return np.full(shape, code, np.uint8)


def test_constant_values_give_that_constant():
    wl = _wl(4, [300], Hq=4, Hkv=2, kmax=5, shuffled_pages=True)
    inp = synth.make_inputs(wl)
    inp["V_pages"] = _constant_codes(inp["V_pages"].shape, 0x5C)   # E4M3 0x5C = 24
    inp["v_scale"] = 0.5
    O = oracle.attn_all(inp)
    assert np.max(np.abs(O - 12.0)) <= 12.0 * 1e-13   # sum(w*12)/sum(w), up to rounding


def test_first_token_of_a_sequence_returns_its_own_value():
    wl = _wl(5, [130, 70], Hq=2, Hkv=1, kmax=3, shuffled_pages=True)
    inp = synth.make_inputs(wl)
    cu, pt = inp["cu_seqlens"], inp["page_table"]
    for b in range(2):
        t = cu[b]
        O = oracle.attn_rows(inp, [t], [1])
        v = inp["V_pages"][pt[b, 0], 0, 0].view(ml_dtypes.float8_e4m3fn).astype(np.float64)
        assert np.array_equal(O[0], v)


def test_equal_scores_average_the_values():
    # k_scale = 0 makes every score 0: O is the plain mean of the query's value rows.
    wl = _wl(6, [200], Hq=2, Hkv=1, kmax=3)
    inp = synth.make_inputs(wl)
    inp["k_scale"] = 0.0
    t, hq = 150, 0   # page 2, position 22 in it
    O = oracle.attn_rows(inp, [t], [hq])[0]
    pages = sorted({int(p) for p in inp["sel_pages"][t, 0] if p >= 0})
    rows = []
    for p in pages:
        for i in range(PAGE):
            if p * PAGE + i <= t:
                rows.append(inp["V_pages"][p, 0, i].view(ml_dtypes.float8_e4m3fn).astype(np.float64))
    assert np.max(np.abs(O - np.mean(rows, axis=0))) < 1e-13


def test_two_key_closed_form():
    # Token 1 selects page 0: keys 0 and 1.  q = 2 e0, k0 = e0, k1 = 0, sm_scale = ln(3)/2:
    # scores ln 3 and 0, weights 3:1, so O = (3 v0 + v1) / 4 = (3*1 + (-1)) / 4 = 0.5 in dim 0.
    inp = {
        "Q": np.zeros((2, 1, D), np.uint16),
        "K_pages": np.zeros((1, 1, PAGE, D), np.uint8),
        "V_pages": np.zeros((1, 1, PAGE, D), np.uint8),
        "page_table": np.zeros((1, 1), np.int32),
        "cu_seqlens": np.array([0, 2], np.int32),
        "sel_pages": np.array([[[0]], [[0]]], np.int32),
        "k_scale": 1.0, "v_scale": 1.0, "sm_scale": math.log(3.0) / 2.0,
    }
    inp["Q"][1, 0, 0] = 0x4000          # bf16 2.0
    inp["K_pages"][0, 0, 0, 0] = 0x38    # E4M3 1.0
    inp["V_pages"][0, 0, 0, 0] = 0x38    # +1
    inp["V_pages"][0, 0, 1, 0] = 0xB8    # -1
    O = oracle.attn_rows(inp, [1], [0])[0]
    assert abs(O[0] - 0.5) < 1e-15 and np.all(O[1:] == 0)


def test_empty_support_gives_zero_output():
    wl = _wl(7, [100], Hq=2, Hkv=1, kmax=3)
    inp = synth.make_inputs(wl)
    inp["sel_pages"][70] = -1
    O = oracle.attn_rows(inp, [70, 70], [0, 1])
    assert np.all(O == 0)


@pytest.mark.parametrize("W,g", [(8, 8), (32, 8), (64, 8), (16, 1), (24, 3)])
def test_grouping_never_changes_a_query_output(W, g):
    wl = _wl(8, [320, 200], Hq=4, Hkv=2, kmax=6, selection="community", communities=3,
             shuffled_pages=True)
    inp = synth.make_inputs(wl)
    direct = oracle.attn_all(inp)
    gr = oracle.group(inp["sel_pages"], inp["cu_seqlens"], W, g)
    via_groups = oracle.attn_grouped(inp, gr)
    assert np.array_equal(direct, via_groups)


def test_physical_page_placement_does_not_matter():
    wl = _wl(9, [260, 130], Hq=2, Hkv=2, kmax=4, shuffled_pages=True)
    inp = synth.make_inputs(wl)
    O1 = oracle.attn_all(inp)
    rng = np.random.default_rng(0)
    perm = rng.permutation(inp["n_phys"])      # move physical page i to slot perm[i]
    inp2 = dict(inp)
    inp2["K_pages"] = np.empty_like(inp["K_pages"])
    inp2["V_pages"] = np.empty_like(inp["V_pages"])
    inp2["K_pages"][perm] = inp["K_pages"]
    inp2["V_pages"][perm] = inp["V_pages"]
    pt = inp["page_table"].copy()
    pt[pt >= 0] = perm[pt[pt >= 0]]
    inp2["page_table"] = pt
    assert np.array_equal(O1, oracle.attn_all(inp2))
