"""pw_attn on the GPU against the oracle, element by element.

Small cases compare every output row; the benchmark workloads at full size compare every row
(workloads 1-2) or, on workloads 3-5, rows the oracle computes one by one: one row of every
group plus every row of the longest unions and of each persistent CTA's first and last group
(parity.sample_rows), always in the same launch configuration the benchmark times (pw_group
then pw_attn on one stream).
"""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_pw_b200 import api, synth
from oracle import oracle

import parity

pytestmark = pytest.mark.gpu


def _run(inp, W, g):
    d = api.device_inputs(inp)
    status = api.new_status()
    O, gr = api.prefill(d["Q"], d["K_pages"], d["V_pages"], d["page_table"], d["sel_pages"],
                        d["cu_seqlens"], d["cu_seqlens_host"], W, g, k_scale=d["k_scale"],
                        v_scale=d["v_scale"], sm_scale=d["sm_scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return O.view(torch.int16).cpu().numpy().view(np.uint16), gr


def _small(seed, seqlens, Hq, Hkv, kmax, selection="uniform", **kw):
    return synth.Workload(f"gpu-attn{seed}", 400 + seed, tuple(seqlens), Hq=Hq, Hkv=Hkv,
                          kmax=kmax, selection=selection, **kw)


SMALL = [
    # (workload, W, g): ragged batch, GQA 3, tile of 24 rows
    (_small(1, [200, 64, 1, 130], 6, 2, 5, shuffled_pages=True), 16, 8),
    # 64-row tiles, several union pages
    (_small(2, [1024], 8, 1, 6, "fixed2"), 32, 8),
    # full 128-row tile (g=16, G=8)
    (_small(3, [512], 16, 2, 6, "community", communities=3), 32, 16),
    # one query per group, contiguous groups
    (_small(4, [300, 77], 4, 1, 8), 1, 1),
    (_small(5, [300, 77], 4, 2, 8, shuffled_pages=True), 8, 8),
    # ragged tails and long unions (every earlier page selected)
    (_small(6, [70, 129, 300], 4, 1, 8), 24, 8),
    (_small(7, [2048], 8, 1, 32, "uniform"), 64, 8),
    # tile rows not a multiple of 32 and g not a power of two
    (_small(8, [450], 10, 2, 7, "community", communities=2), 30, 6),
    # G = 4 with sixteen queries per group: a full 64-row tile on the pipelined kernel
    (_small(18, [1500, 333], 8, 2, 10, "community", communities=4), 64, 16),
]


@pytest.mark.parametrize("wl,W,g", SMALL)
def test_attn_matches_oracle_small(wl, W, g):
    inp = parity.inputs(wl)
    got, _ = _run(inp, W, g)
    ref = oracle.attn_all(inp)
    parity.compare_rows(got.reshape(-1, 128), ref.reshape(-1, 128), wl.name)


def test_dense_causal_selection_long_unions():
    # Every token selects all of its causal pages: unions of up to 32 pages, the running max
    # moves often, so the lazy rescale of O is exercised.
    T, Hkv = 2048, 1
    wl = _small(9, [T], 8, Hkv, 32)
    inp = dict(parity.inputs(wl))
    sel = np.full((T, Hkv, 32), -1, np.int32)
    for t in range(T):
        o = t // 64
        sel[t, 0, : o + 1] = np.arange(o + 1)
    inp["sel_pages"] = sel
    got, _ = _run(inp, 64, 8)
    parity.compare_rows(got.reshape(-1, 128), oracle.attn_all(inp).reshape(-1, 128), "dense")


@pytest.mark.parametrize("qscale", [1e-6, 1.0, 3000.0])
def test_query_magnitudes_and_scales(qscale):
    wl = _small(10, [640, 200], 8, 2, 6, shuffled_pages=True)
    inp = dict(parity.inputs(wl))
    q = torch.from_numpy(inp["Q"].view(np.int16)).view(torch.bfloat16).float() * qscale
    inp["Q"] = q.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    inp["k_scale"], inp["v_scale"] = 0.75, 1.5
    inp["sm_scale"] = inp["sm_scale"] / max(qscale, 1.0) ** 0.5
    got, _ = _run(inp, 32, 8)
    parity.compare_rows(got.reshape(-1, 128), oracle.attn_all(inp).reshape(-1, 128),
                        f"qscale {qscale}")


def test_empty_selections_give_zero_rows():
    wl = _small(11, [300], 4, 1, 6)
    inp = dict(parity.inputs(wl))
    sel = inp["sel_pages"].copy()
    sel[100:140] = -1          # 40 tokens select nothing
    inp["sel_pages"] = sel
    got, _ = _run(inp, 32, 8)
    assert np.all(got.reshape(wl.T, wl.Hq, 128)[100:140] == 0)
    parity.compare_rows(got.reshape(-1, 128), oracle.attn_all(inp).reshape(-1, 128), "empty")


@pytest.mark.parametrize("cfg,W", [(1, 32), (2, 64)])
def test_attn_full_workload_every_row(cfg, W):
    wl = synth.WORKLOADS[cfg]
    inp = parity.inputs(wl)
    got, _ = _run(inp, W, wl.g)
    ref = oracle.attn_all(inp)
    parity.compare_rows(got.reshape(-1, 128), ref.reshape(-1, 128), wl.name)


@pytest.mark.parametrize("cfg,W,g", [(3, 128, 8), (3, 8, 8), (3, 128, 1), (3, 128, 16),
                                     (4, 128, 8), (4, 256, 8), (5, 128, 8)])
def test_attn_full_workload_sampled_rows(cfg, W, g):
    wl = synth.WORKLOADS[cfg]
    inp = parity.inputs(wl)
    got, gr = _run(inp, W, g)
    gh = gr.to_host()
    parity.assert_groups_equal(gh, parity.oracle_groups(wl, W, g))
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    rt, rh = parity.sample_rows(wl, gh, n_random=3000, seed=cfg, n_ctas=n_sm)
    ref = oracle.attn_rows(inp, rt, rh)
    got = got.reshape(wl.T, wl.Hq, 128)[rt, rh]
    max_abs, rel = parity.compare_rows(got, ref, f"{wl.name} W={W} g={g}")
    print(f"{wl.name} W={W} g={g}: {len(rt)} rows of {wl.T * wl.Hq}, every group covered, "
          f"max_abs {max_abs:.3e}, rel_l2 {rel:.3e}")


@pytest.mark.parametrize("code", [0x01, 0x03, 0x07, 0x87, 0x08])
def test_subnormal_and_tiny_values_stay_exact(code):
    # E4M3 subnormals (exponent field 0: m/8 * 2^-6) must survive the decode and the tensor
    # cores: with every V entry equal to one code, each output row is exactly that value.
    wl = _small(12, [300], 4, 1, 6)
    inp = dict(parity.inputs(wl))
    inp["V_pages"] = np.full_like(inp["V_pages"], code)
    got, _ = _run(inp, 32, 8)
    want = oracle.e4m3_to_f64(np.array([code], np.uint8))[0]
    vals = oracle.bf16_bits_to_f64(got)
    assert np.all(vals == want), (code, np.unique(vals)[:5], want)


def test_subnormal_keys():
    # Keys made only of subnormal codes: scores are tiny but not zero, and must match.
    wl = _small(13, [400], 8, 2, 6)
    inp = dict(parity.inputs(wl))
    rng = np.random.default_rng(5)
    K = rng.integers(0, 8, size=inp["K_pages"].shape, dtype=np.uint8)   # codes 0x00..0x07
    K |= (rng.integers(0, 2, size=K.shape, dtype=np.uint8) << 7)        # random sign
    inp["K_pages"] = K
    inp["sm_scale"] = 4000.0    # make the tiny scores matter
    got, _ = _run(inp, 32, 8)
    parity.compare_rows(got.reshape(-1, 128), oracle.attn_all(inp).reshape(-1, 128), "subnormal K")


@pytest.mark.parametrize("scale", [40.0, 400.0])
def test_frequent_rescales(scale):
    # A large softmax scale spreads the scores over tens of binades, so the running max of
    # most rows is raised on many pages and the accumulator rescale runs often.
    wl = _small(14, [1024, 300], 8, 2, 12, "community", communities=3)
    inp = dict(parity.inputs(wl))
    inp["sm_scale"] = inp["sm_scale"] * scale
    got, _ = _run(inp, 64, 8)
    parity.compare_rows(got.reshape(-1, 128), oracle.attn_all(inp).reshape(-1, 128),
                        f"scale {scale}")


def test_q_rows_with_wide_dynamic_range():
    # Q elements spread over 18 binades within every row, so part of each row lies below 2^-9
    # of the row's largest, where the kernel's two-part E4M3 form of Q is not exact; the
    # scores still depend on those elements.
    wl = _small(15, [640, 200], 8, 2, 6, shuffled_pages=True)
    inp = dict(parity.inputs(wl))
    q = torch.from_numpy(inp["Q"].view(np.int16)).view(torch.bfloat16).float()
    gen = torch.Generator().manual_seed(15)
    q = q * torch.pow(2.0, torch.randint(-14, 4, q.shape, generator=gen).float())
    inp["Q"] = q.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got, _ = _run(inp, 32, 8)
    parity.compare_rows(got.reshape(-1, 128), oracle.attn_all(inp).reshape(-1, 128), "wide Q rows")


def _attn_raw(d, groups, max_pages, page_table, status):
    """pw_attn straight through the C ABI (no binding-side checks), on the current stream."""
    import ctypes as C
    from dynamic_sparse_attention_pw_b200 import _lib
    L = _lib.load()
    Q = d["Q"]
    T, Hq, _ = Q.shape
    O = torch.zeros_like(Q)
    st = groups.struct()
    p = lambda t: C.c_void_p(t.data_ptr())
    rc = L.pw_attn(p(Q), p(d["K_pages"]), p(d["V_pages"]), p(page_table), max_pages,
                   d["K_pages"].shape[0], p(d["cu_seqlens"]), d["cu_seqlens"].numel() - 1, T, Hq,
                   d["K_pages"].shape[1], 1.0, 1.0, float(d["sm_scale"]), C.byref(st), p(O),
                   p(status), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, int(status.item())


def test_page_table_narrower_than_a_sequence_is_reported():
    # The caller passes a page table with one column fewer than the sequence has pages: the
    # kernel must not index past the row (the last page's id equals the row's width); it
    # records PW_ERR_INVALID_ARG in the device status.  Every access stays inside the buffers.
    wl = _small(16, [256], 4, 1, 4)
    d = api.device_inputs(parity.inputs(wl))
    status = api.new_status()
    groups = api.pw_group(d["sel_pages"], d["cu_seqlens"], d["cu_seqlens_host"], 32, 8, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    pt = d["page_table"]
    assert pt.shape == (1, 4)
    rc, code = _attn_raw(d, groups, pt.shape[1] - 1, pt, status)
    assert rc == 0 and code == 1, (rc, code)        # PW_ERR_INVALID_ARG


def test_page_table_entry_outside_the_pool_is_reported():
    # A page table entry outside [0, n_phys) records PW_ERR_INVALID_ARG; the kernel reads slot
    # 0 in its place, so nothing outside the K and V pools is read.
    wl = _small(17, [256, 130], 4, 1, 4, shuffled_pages=True)
    d = api.device_inputs(parity.inputs(wl))
    status = api.new_status()
    groups = api.pw_group(d["sel_pages"], d["cu_seqlens"], d["cu_seqlens_host"], 32, 8, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    pt = d["page_table"].clone()
    pt[1, 1] = d["K_pages"].shape[0]                  # one past the pool
    rc, code = _attn_raw(d, groups, pt.shape[1], pt, status)
    assert rc == 0 and code == 1, (rc, code)
