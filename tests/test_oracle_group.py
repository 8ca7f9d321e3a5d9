"""Pins of the oracle's bounded-window greedy grouping.

The grouping is a heuristic (AI Radio episode on "PageWeaver: KV-Guided Query Unions for
Sparse Attention", paper summary: queries whose selected sets add few new pages are collected
greedily inside a bounded window; the execution size g is fixed independently of W).  It is
pinned by hand-derived examples, special cases with known answers, invariants, and a check
of the greedy-choice conditions on every step the oracle took.
"""
import json
import os

import numpy as np
import pytest

from dynamic_sparse_attention_pw_b200 import synth
from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PAGE = 64


def _load():
    with open(os.path.join(GOLDEN, "group_hand_examples.json")) as f:
        return {e["name"][0]: e for e in json.load(f)["examples"]}


def _sel_from_sets(T, Hkv, kmax, sets_of):
    sel = np.full((T, Hkv, kmax), -1, np.int32)
    for t in range(T):
        for h in range(Hkv):
            s = sets_of(t, h)
            sel[t, h, : len(s)] = s
    return sel


def _groups_as_lists(gr):
    out = []
    for i in range(gr["n_groups"]):
        n = gr["gsize"][i]
        mem = [int(x) for x in gr["qids"][i, :n]]
        un = [int(x) for x in gr["union_pages"][gr["union_off"][i]: gr["union_off"][i + 1]]]
        po = [int(x) for x in gr["order"][i, :n]] if "order" in gr else None
        out.append((mem, un, po, [int(x) for x in gr["gmeta"][i]]))
    return out


def test_hand_example_A_window_greedy():
    ex = _load()["A"]
    T, kmax = ex["seqlens"][0], ex["kmax"]
    first = ex["window_sets"]["first_token"]
    sets = ex["window_sets"]["sets"]
    sel = _sel_from_sets(T, 1, kmax, lambda t, h: sets[t - first] if t >= first else [t // PAGE])
    gr = oracle.group(sel, synth.cu_seqlens_of(ex["seqlens"]), ex["W"], ex["g"], with_order=True)
    assert gr["status"] == 0
    gl = _groups_as_lists(gr)
    # prefix rule: contiguous groups of 4 with union = own page
    for w in range(first // ex["W"]):
        for j in range(2):
            mem, un, po, meta = gl[2 * w + j]
            lo = ex["W"] * w + 4 * j
            assert mem == list(range(lo, lo + 4))
            assert un == [lo // PAGE]
            assert meta == [0, 0, w]
    tail = gl[2 * (first // ex["W"]):]
    assert len(tail) == 2
    for (mem, un, po, meta), exp in zip(tail, ex["expected_window_groups"]):
        assert mem == exp["members"]
        assert un == exp["union"]
        assert po == exp["pick_order"]


def test_hand_example_C_heads_group_independently():
    ex = _load()["C"]
    T, Hkv, kmax = ex["seqlens"][0], ex["Hkv"], ex["kmax"]
    first = ex["window_sets_per_head"]["first_token"]
    sets = ex["window_sets_per_head"]["sets"]
    sel = _sel_from_sets(T, Hkv, kmax, lambda t, h: sets[h][t - first] if t >= first else [0])
    gr = oracle.group(sel, synth.cu_seqlens_of(ex["seqlens"]), ex["W"], ex["g"], with_order=True)
    gl = _groups_as_lists(gr)
    per_head = len(gl) // Hkv
    assert per_head == 34
    for h in range(Hkv):
        mine = gl[h * per_head:(h + 1) * per_head]
        for i in range(32):
            mem, un, po, meta = mine[i]
            assert mem == [2 * i, 2 * i + 1] and un == [0] and meta == [0, h, i // 2]
        for (mem, un, po, meta), exp in zip(mine[32:], ex["expected_window_groups_per_head"][h]):
            assert (mem, un, po) == (exp["members"], exp["union"], exp["pick_order"])
            assert meta == [0, h, 16]


def test_hand_example_D_ragged_batch_and_empty_unions():
    ex = _load()["D"]
    sets = ex["sets"]
    T = sum(ex["seqlens"])
    sel = _sel_from_sets(T, 1, ex["kmax"], lambda t, h: sets[t])
    gr = oracle.group(sel, synth.cu_seqlens_of(ex["seqlens"]), ex["W"], ex["g"])
    gl = _groups_as_lists(gr)
    assert len(gl) == len(ex["expected_groups"])
    for (mem, un, _, meta), exp in zip(gl, ex["expected_groups"]):
        assert mem == exp["members"] and un == exp["union"] and meta == exp["meta"]


# ------------------------------------------------------------------------------------------
# special cases with a known answer
# ------------------------------------------------------------------------------------------

def _small(seed_id, seqlens, Hkv=2, kmax=6, selection="uniform", **kw):
    return synth.Workload(f"small{seed_id}", 100 + seed_id, tuple(seqlens), Hq=Hkv * 2, Hkv=Hkv,
                          kmax=kmax, selection=selection, **kw)


@pytest.mark.parametrize("g", [1, 4, 8])
def test_window_equal_to_g_is_contiguous_grouping(g):
    wl = _small(1, [300, 77, 512], selection="uniform")
    sel = synth.make_selection(wl)
    cu = synth.cu_seqlens_of(wl.seqlens)
    gr = oracle.group(sel, cu, W=g, g=g)
    i = 0
    for b, n in enumerate(wl.seqlens):
        for h in range(wl.Hkv):
            for lo in range(0, n, g):
                mem = list(gr["qids"][i, : gr["gsize"][i]])
                assert mem == list(range(cu[b] + lo, cu[b] + min(lo + g, n)))
                i += 1
    assert i == gr["n_groups"]


def test_g1_gives_singletons_in_token_order():
    wl = _small(2, [130, 64], selection="uniform")
    sel = synth.make_selection(wl)
    gr = oracle.group(sel, synth.cu_seqlens_of(wl.seqlens), W=32, g=1)
    assert np.all(gr["gsize"] == 1)
    # order: (b, h, window, seed) -> within (b,h) tokens ascending
    i = 0
    cu = synth.cu_seqlens_of(wl.seqlens)
    for b, n in enumerate(wl.seqlens):
        for h in range(wl.Hkv):
            assert list(gr["qids"][i:i + n, 0]) == list(range(cu[b], cu[b] + n))
            assert np.all(gr["gmeta"][i:i + n, 1] == h)
            i += n
    assert i == gr["n_groups"]


def test_identical_sets_give_contiguous_groups_for_any_window():
    T, Hkv, kmax = 256, 1, 3
    sel = _sel_from_sets(T, Hkv, kmax, lambda t, h: [0])
    gr = oracle.group(sel, np.array([0, T], np.int32), W=64, g=8)
    assert gr["n_groups"] == 32
    for i in range(32):
        assert list(gr["qids"][i]) == list(range(8 * i, 8 * i + 8))


def test_two_interleaved_communities_are_separated():
    # Tokens alternate between two disjoint page sets (the pages' observation that adjacent
    # query groups mix two page communities): contiguous groups take both, a window of 16
    # separates them, so each group's union is one community plus nothing else.
    T = 128 + 16
    A, Bc = [0, 2], [1]
    sel = _sel_from_sets(T, 1, 2, lambda t, h: (A if t % 2 == 0 else Bc) if t >= 128 else [t // 64])
    cu = np.array([0, T], np.int32)
    contig = oracle.group(sel, cu, W=8, g=8)
    regrp = oracle.group(sel, cu, W=16, g=8)
    c = _groups_as_lists(contig)[-2:]
    r = _groups_as_lists(regrp)[-2:]
    assert c[0][1] == [0, 1, 2] and c[1][1] == [0, 1, 2]
    assert r[0][0] == list(range(128, 144, 2)) and r[0][1] == [0, 2]
    assert r[1][0] == list(range(129, 144, 2)) and r[1][1] == [1]


# ------------------------------------------------------------------------------------------
# invariants and the greedy-choice conditions, on random inputs
# ------------------------------------------------------------------------------------------

def _sets(sel, t, h):
    return {int(p) for p in sel[t, h] if p >= 0}


CASES = [
    (_small(3, [200, 64, 1, 333]), 32, 8),
    (_small(4, [512], Hkv=1, kmax=4, selection="fixed2"), 64, 8),
    (_small(5, [1024], Hkv=2, kmax=8, selection="community", communities=4), 128, 8),
    (_small(6, [700, 129], Hkv=3, kmax=5, selection="uniform"), 24, 3),
    (_small(7, [256], Hkv=1, kmax=16, selection="uniform"), 256, 8),
]


@pytest.mark.parametrize("wl,W,g", CASES)
def test_invariants_and_greedy_conditions(wl, W, g):
    sel = synth.make_selection(wl)
    # sprinkle duplicates: repeating a page must not change anything (set semantics)
    sel2 = sel.copy()
    dup = sel2[:, :, 0:1]
    free = sel2[:, :, -1] < 0
    sel2[:, :, -1] = np.where(free, dup[:, :, 0], sel2[:, :, -1])
    cu = synth.cu_seqlens_of(wl.seqlens)
    gr = oracle.group(sel, cu, W, g, with_order=True)
    gr2 = oracle.group(sel2, cu, W, g, with_order=True)
    assert gr["status"] == 0 and gr2["status"] == 0
    for key in ("qids", "gsize", "gmeta", "union_off", "union_pages"):
        assert np.array_equal(gr[key], gr2[key]), key
    n_expected, _ = oracle.group_counts(cu, wl.Hkv, wl.kmax, W, g)
    assert gr["n_groups"] == n_expected
    seen = np.zeros((wl.T, wl.Hkv), np.int32)
    for i in range(gr["n_groups"]):
        b, h, w = gr["gmeta"][i]
        n = gr["gsize"][i]
        assert 1 <= n <= g
        mem = gr["qids"][i, :n]
        assert np.all(gr["qids"][i, n:] == -1)
        assert np.all(np.diff(mem) > 0)
        lo, hi = cu[b] + w * W, min(cu[b] + (w + 1) * W, cu[b + 1])
        assert np.all((mem >= lo) & (mem < hi))
        seen[mem, h] += 1
        un = gr["union_pages"][gr["union_off"][i]: gr["union_off"][i + 1]]
        assert np.all(np.diff(un) > 0)
        assert set(int(p) for p in un) == set().union(*[_sets(sel, t, h) for t in mem])
        # greedy-choice conditions on the recorded pick order
        order = [int(x) for x in gr["order"][i, :n]]
        assert sorted(order) == list(mem)
        # candidates still unassigned when this group started: tokens of the window not in
        # an earlier group of the same (b, h, w)
        earlier = set()
        j = i - 1
        while j >= 0 and tuple(gr["gmeta"][j]) == (b, h, w):
            earlier |= set(int(x) for x in gr["qids"][j, : gr["gsize"][j]])
            j -= 1
        remaining = [t for t in range(lo, hi) if t not in earlier]
        assert order[0] == min(remaining)
        U = set(_sets(sel, order[0], h))
        remaining.remove(order[0])
        for c in order[1:]:
            cost = {r: len(_sets(sel, r, h) - U) for r in remaining}
            best = min(cost.values())
            assert cost[c] == best
            assert c == min(r for r in remaining if cost[r] == best)
            U |= _sets(sel, c, h)
            remaining.remove(c)
        if n < g:
            assert not remaining  # a group stops short only when its window is exhausted
    assert np.all(seen == 1)  # every query assigned exactly once per kv head


def test_bad_selection_is_rejected():
    wl = _small(8, [128], Hkv=1, kmax=4)
    sel = synth.make_selection(wl)
    cu = synth.cu_seqlens_of(wl.seqlens)
    assert oracle.validate(sel, cu) == 0
    bad = sel.copy()
    bad[10, 0, 3] = 1  # token 10 sits on page 0: page 1 is in its future
    assert oracle.validate(bad, cu) == 3
    assert oracle.group(bad, cu, 32, 8)["status"] == 3
    bad = sel.copy()
    bad[100, 0, 2] = -2
    assert oracle.validate(bad, cu) == 3
