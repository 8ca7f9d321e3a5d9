"""Page-pair formulation of the union attention (a direct KV-page union), as a numpy model:
used to check that the decomposition is exact and to count its work on the benchmark
selections beside the query unions.  Test infrastructure; nothing in the package imports it.

Reading of the pages ("PageWeaver: KV-Guided Query Unions for Sparse Attention", Abstract: a
direct KV-page union implementation gives a complementary study of nonlocal reuse and reduction
cost; AI Radio episode on the paper, paper summary: disjoint page pairs and full membership
form common or exclusive query lists):
  - per (sequence b, kv head h) the pages are paired as (2i, 2i+1);
  - for each pair, the queries that selected both pages form its common list and those that
    selected exactly one its two exclusive lists; each list, in token order, is cut into tiles
    of at most g queries;
  - a tile reads its one or two pages once and gives each of its rows a partial (m, l, acc)
    over the keys of those pages that the row may see (its position and before, inside the
    sequence);
  - a query's output merges its partials over the pairs it touched:
    O = sum_i e^(m_i - M) acc_i / sum_i e^(m_i - M) l_i, M = max_i m_i.

Run as a script it prints the counts of the design study for workloads 3, 4 and 5.
"""
import ml_dtypes
import numpy as np

PAGE = 64
D = 128


def _membership(sel_rows, n_tokens):
    """Token x page membership of one (sequence, kv head), padded to an even page count."""
    P = (n_tokens + PAGE - 1) // PAGE
    M = np.zeros((n_tokens, P + (P & 1)), bool)
    r, c = np.nonzero(sel_rows >= 0)
    M[r, sel_rows[r, c]] = True
    return M


def pair_tiles(sel, cu, g):
    """Tiles (b, h, pages, member tokens) in a fixed order: sequences, kv heads, pairs, then the
    common list and the two exclusive lists, each cut into runs of at most g tokens."""
    tiles = []
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        if e == s:
            continue
        for h in range(sel.shape[1]):
            M = _membership(sel[s:e, h], e - s)
            for i in range(0, M.shape[1], 2):
                a, c = M[:, i], M[:, i + 1]
                for pages, who in (((i, i + 1), a & c), ((i,), a & ~c), ((i + 1,), ~a & c)):
                    toks = s + np.nonzero(who)[0]
                    for k0 in range(0, len(toks), g):
                        tiles.append((b, h, pages, toks[k0:k0 + g]))
    return tiles


def pair_counts(sel, cu, G, g):
    """(two-page tiles, one-page tiles, page loads, partial rows) without listing the tiles."""
    tiles2 = tiles1 = partial_rows = 0
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        if e == s:
            continue
        for h in range(sel.shape[1]):
            M = _membership(sel[s:e, h], e - s)
            a, c = M[:, 0::2], M[:, 1::2]
            tiles2 += int(((( a & c).sum(0) + g - 1) // g).sum())
            tiles1 += int(((( a & ~c).sum(0) + g - 1) // g).sum())
            tiles1 += int((((~a & c).sum(0) + g - 1) // g).sum())
            partial_rows += int((a | c).sum()) * G
    return tiles2, tiles1, 2 * tiles2 + tiles1, partial_rows


def page_pair_attention(inp, g):
    """O (binary64) [T, Hq, 128] by the page-pair decomposition and the cross-pair merge."""
    Q = inp["Q"].view(ml_dtypes.bfloat16).astype(np.float64)
    K = inp["K_pages"].view(ml_dtypes.float8_e4m3fn).astype(np.float64) * inp["k_scale"]
    V = inp["V_pages"].view(ml_dtypes.float8_e4m3fn).astype(np.float64) * inp["v_scale"]
    sel, cu, pt = inp["sel_pages"], inp["cu_seqlens"], inp["page_table"]
    T, Hq, _ = Q.shape
    G = Hq // sel.shape[1]
    parts = {}
    for b, h, pages, toks in pair_tiles(sel, cu, g):
        s, e = int(cu[b]), int(cu[b + 1])
        pos_k = np.concatenate([p * PAGE + np.arange(PAGE) for p in pages])
        pos_k = pos_k[pos_k < e - s]
        phys = pt[b, pos_k // PAGE]
        Kd, Vd = K[phys, h, pos_k % PAGE], V[phys, h, pos_k % PAGE]
        for t in toks:
            seen = pos_k <= t - s
            for j in range(G):
                hq = h * G + j
                S = np.where(seen, (Kd @ Q[t, hq]) * inp["sm_scale"], -np.inf)
                m = S.max()
                w = np.exp(S - m)
                parts.setdefault((int(t), hq), []).append((m, w.sum(), w @ Vd))
    O = np.zeros((T, Hq, D))
    for (t, hq), lst in parts.items():
        M = max(p[0] for p in lst)
        num = sum(np.exp(p[0] - M) * p[2] for p in lst)
        den = sum(np.exp(p[0] - M) * p[1] for p in lst)
        O[t, hq] = num / den
    return O


def main():
    import sys
    import os
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from dynamic_sparse_attention_pw_b200 import synth
    from oracle import oracle
    hbm = 6549.4e9
    for cfg in (3, 4, 5):
        wl = synth.WORKLOADS[cfg]
        inp = synth.make_inputs(wl)
        gr = oracle.group(inp["sel_pages"], inp["cu_seqlens"], 128, 8)
        qu_pages = int(np.diff(gr["union_off"]).sum())
        t2, t1, pp_pages, rows = pair_counts(inp["sel_pages"], inp["cu_seqlens"], wl.G, 8)
        merge = rows * (D * 4 + 8) * 2
        print(f"workload {cfg}: query unions {gr['n_groups']} tiles, {qu_pages * 16384 / 1e9:.2f} GB"
              f" of pages ({qu_pages * 16384 / hbm * 1e3:.2f} ms); page pairs {t2} + {t1} tiles,"
              f" {pp_pages * 16384 / 1e9:.2f} GB of pages, {merge / 1e9:.1f} GB of partials"
              f" ({(pp_pages * 16384 + merge) / hbm * 1e3:.2f} ms)")


if __name__ == "__main__":
    main()
