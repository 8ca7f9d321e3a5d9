"""Shared helpers of the GPU parity tests: cached synthetic inputs and the comparisons.

Tolerance (stated by the method's acceptance bar): group IDs and union lists bit-exact; O
within max-abs 2e-2 and rel-L2 1e-3 of the oracle rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import functools

import numpy as np

from dynamic_sparse_attention_pw_b200 import synth
from oracle import oracle

MAX_ABS = 2e-2
REL_L2 = 1e-3


@functools.lru_cache(maxsize=3)
def inputs(wl: synth.Workload) -> dict:
    return synth.make_inputs(wl)


@functools.lru_cache(maxsize=8)
def oracle_groups(wl: synth.Workload, W: int, g: int) -> dict:
    inp = inputs(wl)
    gr = oracle.group(inp["sel_pages"], inp["cu_seqlens"], W, g)
    assert gr["status"] == 0
    return gr


def assert_groups_equal(got: dict, ref: dict):
    assert got["n_groups"] == ref["n_groups"]
    for key in ("gsize", "gmeta", "qids", "union_off", "union_pages"):
        a, b = np.asarray(got[key]), np.asarray(ref[key])
        assert a.shape == b.shape, (key, a.shape, b.shape)
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            raise AssertionError(f"{key} differs at {bad[:5].tolist()} "
                                 f"(got {a[tuple(bad[0])]}, want {b[tuple(bad[0])]})")


def compare_rows(got_bits: np.ndarray, ref_f64: np.ndarray, what: str = ""):
    """got_bits: bf16 bits [n, 128] from the GPU; ref_f64: oracle binary64 [n, 128]."""
    got = oracle.bf16_bits_to_f64(got_bits)
    ref = oracle.bf16_bits_to_f64(oracle.f64_to_bf16(ref_f64))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / denom) if denom > 0 else float(np.linalg.norm(got))
    assert max_abs <= MAX_ABS and rel <= REL_L2, \
        f"{what}: max_abs {max_abs:.3e} (<= {MAX_ABS}), rel_l2 {rel:.3e} (<= {REL_L2})"
    return max_abs, rel


def sample_rows(wl: synth.Workload, groups: dict, n_random: int, seed: int = 0,
                n_ctas: int = 148, n_largest: int = 64):
    """(t, hq) rows to compare at full size, chosen so that every group and every place where a
    pipelined kernel changes state is covered:
      - one row (random member, random head) of every group, so every group's union, page
        steps and odd page counts are exercised;
      - every row of the n_largest groups with the longest unions;
      - every row of the first and the last n_ctas groups: where the persistent kernel's CTAs
        start and finish, both for a single sequence (CTA i walks i, i + n_ctas, ...) and for a
        ragged batch (CTAs take groups from a counter, the last group first);
      - every row of the first, a middle and the last group;
      - n_random uniformly drawn rows."""
    rng = np.random.default_rng(seed)
    G = wl.G
    n = groups["n_groups"]
    gsize = np.asarray(groups["gsize"][:n])
    qids = np.asarray(groups["qids"][:n])
    heads = np.asarray(groups["gmeta"][:n, 1])
    usize = np.diff(np.asarray(groups["union_off"][: n + 1]))
    rows = set()
    if n > 0:
        mem = (rng.random(n) * gsize).astype(np.int64)
        hqs = heads * G + rng.integers(0, G, n)
        for t, hq in zip(qids[np.arange(n), mem], hqs):
            rows.add((int(t), int(hq)))
    full = set([0, n // 2, n - 1] if n > 0 else [])
    full.update(int(i) for i in np.argsort(-usize, kind="stable")[:n_largest])
    c = min(n_ctas, n)
    full.update(range(c))
    full.update(range(max(n - c, 0), n))
    for gi in full:
        h = int(heads[gi])
        for t in qids[gi, : gsize[gi]]:
            for j in range(G):
                rows.add((int(t), h * G + j))
    for t, hq in zip(rng.integers(0, wl.T, n_random), rng.integers(0, wl.Hq, n_random)):
        rows.add((int(t), int(hq)))
    rows = sorted(rows)
    return np.array([r[0] for r in rows], np.int64), np.array([r[1] for r in rows], np.int32)
