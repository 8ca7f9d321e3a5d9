"""pw_group on the GPU against the oracle: group IDs and union lists bit-exact."""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_pw_b200 import api, synth
from oracle import oracle

import parity

pytestmark = pytest.mark.gpu


def _gpu_groups(wl, W, g, sel=None):
    inp = parity.inputs(wl)
    sel = inp["sel_pages"] if sel is None else sel
    dev_sel = torch.from_numpy(np.ascontiguousarray(sel)).cuda()
    cu = torch.from_numpy(inp["cu_seqlens"]).cuda()
    status = api.new_status()
    gr = api.pw_group(dev_sel, cu, inp["cu_seqlens"], W, g, status=status)
    torch.cuda.synchronize()
    return gr, int(status.item())


def _small(seed, seqlens, Hq, Hkv, kmax, selection="uniform", **kw):
    return synth.Workload(f"gpu-group{seed}", 300 + seed, tuple(seqlens), Hq=Hq, Hkv=Hkv,
                          kmax=kmax, selection=selection, **kw)


SMALL = [
    (_small(1, [200, 64, 1, 130], 4, 2, 5), 16, 8),
    (_small(2, [1000], 8, 1, 4, "fixed2"), 32, 8),
    (_small(3, [777, 64, 2049], 8, 2, 12, "community", communities=4), 64, 8),
    (_small(4, [4096], 4, 1, 32, "community", communities=8), 256, 8),
    (_small(5, [700, 129], 6, 3, 5), 24, 3),
    (_small(6, [513], 2, 1, 9), 32, 1),
    (_small(7, [2048, 31], 4, 2, 40), 128, 32),
    (_small(8, [70000], 2, 1, 6), 128, 8),         # 1094 pages: two bitset words per lane
    # more than 8 bitset words: windows renumbered to their own pages before the search
    (_small(9, [20000, 3000], 4, 2, 24, "community", communities=8), 64, 8),
    (_small(10, [40000], 2, 1, 16, "community", communities=16), 256, 4),
    # uniform selections: later windows hold more than 256 distinct pages and are staged whole
    (_small(11, [30000, 500], 4, 2, 40), 128, 8),
]


@pytest.mark.parametrize("wl,W,g", SMALL)
def test_group_matches_oracle_small(wl, W, g):
    gr, st = _gpu_groups(wl, W, g)
    assert st == 0
    parity.assert_groups_equal(gr.to_host(), parity.oracle_groups(wl, W, g))


@pytest.mark.parametrize("cfg,W,g", [
    (1, 32, 8), (2, 64, 8), (3, 128, 8), (3, 8, 8), (3, 128, 1),
    (4, 32, 8), (4, 64, 8), (4, 128, 8), (4, 256, 8), (5, 128, 8),
])
def test_group_matches_oracle_benchmark_workloads(cfg, W, g):
    wl = synth.WORKLOADS[cfg]
    gr, st = _gpu_groups(wl, W, g)
    assert st == 0
    parity.assert_groups_equal(gr.to_host(), parity.oracle_groups(wl, W, g))


def test_duplicates_count_once():
    wl = _small(9, [640], 4, 2, 8)
    sel = parity.inputs(wl)["sel_pages"].copy()
    free = sel[:, :, -1] < 0
    sel[:, :, -1] = np.where(free, sel[:, :, 0], sel[:, :, -1])
    gr, st = _gpu_groups(wl, 64, 8, sel=sel)
    assert st == 0
    ref = oracle.group(sel, parity.inputs(wl)["cu_seqlens"], 64, 8)
    parity.assert_groups_equal(gr.to_host(), ref)


def test_bad_selection_sets_device_status():
    wl = _small(10, [256], 2, 1, 4)
    sel = parity.inputs(wl)["sel_pages"].copy()
    sel[10, 0, 3] = 2            # token 10 is on page 0
    gr, st = _gpu_groups(wl, 32, 8, sel=sel)
    assert st == api._lib.PW_ERR_BAD_SELECTION
    sel = parity.inputs(wl)["sel_pages"].copy()
    sel[200, 0, 2] = -7
    gr, st = _gpu_groups(wl, 32, 8, sel=sel)
    assert st == api._lib.PW_ERR_BAD_SELECTION
    # a clean call afterwards resets the status
    gr, st = _gpu_groups(wl, 32, 8)
    assert st == 0
