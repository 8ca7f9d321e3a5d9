"""The page-pair formulation (a direct KV-page union: common and exclusive query lists per
disjoint page pair, partials merged across pairs) reproduces the oracle's output, and its tile
lists cover every selected page of every query exactly once.  CPU only."""
import numpy as np
import pytest

from dynamic_sparse_attention_pw_b200 import synth
from oracle import oracle

import page_pairs


def _wl(seed, seqlens, Hq, Hkv, kmax, selection="uniform", **kw):
    return synth.Workload(f"pairs{seed}", 700 + seed, tuple(seqlens), Hq=Hq, Hkv=Hkv, kmax=kmax,
                          selection=selection, **kw)


CASES = [
    (_wl(1, [200, 64, 1, 130], 6, 2, 5, shuffled_pages=True), 8),   # ragged, odd page counts
    (_wl(2, [300], 8, 1, 4, "fixed2"), 8),
    (_wl(3, [512, 96], 4, 2, 6, "community", communities=3), 4),
    (_wl(4, [257], 4, 1, 12), 3),                                   # long unions, g = 3
]


@pytest.mark.parametrize("wl,g", CASES)
def test_page_pairs_reproduce_the_oracle(wl, g):
    inp = synth.make_inputs(wl)
    ref = oracle.attn_all(inp)
    got = page_pairs.page_pair_attention(inp, g)
    assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


@pytest.mark.parametrize("wl,g", CASES)
def test_every_selected_page_lies_in_exactly_one_tile_of_its_query(wl, g):
    inp = synth.make_inputs(wl)
    sel, cu = inp["sel_pages"], inp["cu_seqlens"]
    seen = {}
    for b, h, pages, toks in page_pairs.pair_tiles(sel, cu, g):
        assert 1 <= len(toks) <= g
        for t in toks:
            mine = set(int(p) for p in sel[t, h] if p >= 0)
            assert set(pages) <= mine          # a tile's pages are all selected by its members
            for p in pages:
                key = (int(t), h, p)
                assert key not in seen
                seen[key] = True
    want = {(int(t), h, int(p)) for t in range(sel.shape[0]) for h in range(sel.shape[1])
            for p in sel[t, h] if p >= 0}
    assert set(seen) == want


@pytest.mark.parametrize("wl,g", CASES)
def test_counts_agree_with_the_tile_lists(wl, g):
    inp = synth.make_inputs(wl)
    tiles = page_pairs.pair_tiles(inp["sel_pages"], inp["cu_seqlens"], g)
    t2 = sum(1 for _, _, pages, _ in tiles if len(pages) == 2)
    t1 = len(tiles) - t2
    rows = sum(len(toks) for _, _, _, toks in tiles) * wl.G
    pairs_touched = rows  # one partial per (query, pair): each query sits in one list per pair
    assert page_pairs.pair_counts(inp["sel_pages"], inp["cu_seqlens"], wl.G, g) == (
        t2, t1, 2 * t2 + t1, pairs_touched)
