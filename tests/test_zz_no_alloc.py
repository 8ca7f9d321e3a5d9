"""pw_group_noalloc: the grouping entry point for callers that cannot allocate device memory
(for example code where cudaMalloc is not allowed, or a plug-in that only receives input and
output buffers).  Its scratch is a fixed device array inside the library.

Checked through the C ABI against the ordinary pw_group (caller-supplied workspace) on two
calls in a row with different inputs, bit-exact (the tolerance of every grouping test), and
for the size limit.  This file is collected last so a failure here cannot hide another test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from dynamic_sparse_attention_pw_b200 import _lib, api, synth

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 * 1024 * 1024


def _noalloc():
    L = _lib.load()
    f = L.pw_group_noalloc
    f.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                  C.POINTER(_lib.PwGroups), C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    return f


def _call_noalloc(sel, cu, cu_host, W, g, groups, status):
    T, Hkv, kmax = sel.shape
    cu_host = np.ascontiguousarray(cu_host, np.int32)
    st = groups.struct()
    return _noalloc()(C.c_void_p(sel.data_ptr()), C.c_void_p(cu.data_ptr()),
                      cu_host.ctypes.data_as(C.c_void_p), len(cu_host) - 1, Hkv, kmax, W, g,
                      C.byref(st), C.c_void_p(status.data_ptr()),
                      C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _case(wl, W, g):
    inp = synth.make_inputs(wl)
    sel = torch.from_numpy(inp["sel_pages"]).cuda()
    cu = torch.from_numpy(inp["cu_seqlens"]).cuda()
    return wl, inp["cu_seqlens"], sel, cu, W, g


def _as_host(groups: "api.Groups", T, Hkv):
    h = groups.to_host()
    h["bits"] = groups.bits[: T * Hkv * groups.words].cpu().numpy()
    return h


def test_noalloc_matches_pw_group_on_two_calls_in_a_row():
    cases = [
        _case(synth.WORKLOADS[2], 64, 8),
        _case(synth.Workload("noalloc-ragged", 77, (700, 129, 2048), Hq=6, Hkv=3, kmax=9,
                             selection="uniform"), 24, 3),
    ]
    got = []
    for wl, cu_host, sel, cu, W, g in cases:       # two calls in a row, different shapes
        T, Hkv, kmax = sel.shape
        groups = api.Groups.allocate(T, Hkv, cu_host, kmax, W, g)
        status = api.new_status()
        code = _call_noalloc(sel, cu, cu_host, W, g, groups, status)
        assert code == _lib.PW_OK, _lib.status_string(code)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got.append(_as_host(groups, T, Hkv))
    for (wl, cu_host, sel, cu, W, g), mine in zip(cases, got):
        T, Hkv, kmax = sel.shape
        ref_groups = api.pw_group(sel, cu, cu_host, W, g)   # caller-supplied workspace
        torch.cuda.synchronize()
        ref = _as_host(ref_groups, T, Hkv)
        assert mine["n_groups"] == ref["n_groups"]
        for key in ("qids", "gsize", "gmeta", "union_off", "union_pages", "bits"):
            assert np.array_equal(mine[key], ref[key]), key


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 32 sequences of 131072 tokens, 8 kv heads: the workspace is far above 32 MiB.
    cu_host = np.arange(33, dtype=np.int32) * 131072
    need = api.pw_groups_size(cu_host, 8, 4, 128, 8)[3]
    assert need > SCRATCH_BYTES
    g = _lib.PwGroups()
    code = _noalloc()(C.c_void_p(16), C.c_void_p(16), cu_host.ctypes.data_as(C.c_void_p), 32, 8,
                      4, 128, 8, C.byref(g), C.c_void_p(16), None)
    assert code == _lib.PW_ERR_CAPACITY
