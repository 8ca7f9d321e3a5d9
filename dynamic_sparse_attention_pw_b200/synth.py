"""Seeded synthetic inputs for the PageWeaver prefill hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no grouping, no attention).  Both the CPU oracle and the
CUDA path consume the exact bytes it returns.

Why synthetic: "PageWeaver: KV-Guided Query Unions for Sparse Attention"
(arXiv 2610.11201, Abstract) measures on six captured page selections that are
not public; the workloads below stand in for them with the shapes, sizes and
page-affinity structure the pages describe (adjacent query groups mix two page
communities while distant queries share them -- AI Radio episode on the paper,
paper summary).

Layouts (all row-major, contiguous):
  cu_seqlens  int32 [B+1]            token offsets of the ragged batch
  sel_pages   int32 [T, Hkv, kmax]   logical page ids selected per (token, kv head), -1 padded
  Q           bf16  [T, Hq, 128]
  K_pages     uint8 [P_phys, Hkv, 64, 128]   FP8 E4M3 codes, physical page order
  V_pages     uint8 [P_phys, Hkv, 64, 128]
  page_table  int32 [B, max_pages]   logical -> physical page, -1 beyond a sequence's pages

Random streams (torch CPU generators seeded from numpy SeedSequence):
  0 = Q, 1 = K, 2 = V, 3 = community assignment, 4 = selection draws, 5 = page table.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

PAGE = 64
HEAD_DIM = 128

STREAM_Q, STREAM_K, STREAM_V, STREAM_COMM, STREAM_SEL, STREAM_PT = range(6)


@dataclass(frozen=True)
class Workload:
    """One synthetic prefill workload.

    selection:
      "fixed2"    -- own page, page 0 and up to kmax-2 pages drawn uniformly from pages 1..o-1
      "community" -- own page, page 0 and up to kmax-2 pages drawn from the token's community
      "uniform"   -- own page and up to kmax-1 pages drawn uniformly from pages 0..o-1
    """
    name: str
    seed_id: int
    seqlens: tuple
    Hq: int
    Hkv: int
    kmax: int
    selection: str
    communities: int = 0
    block: int = 128            # query block that shares one community pair
    shuffled_pages: bool = False
    g: int = 8
    W: int = 32
    k_scale: float = 1.0
    v_scale: float = 1.0
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def T(self) -> int:
        return int(sum(self.seqlens))

    @property
    def B(self) -> int:
        return len(self.seqlens)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(HEAD_DIM)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the benchmark plan, by size.
WORKLOADS = {
    1: Workload("1k-fixed2", 1, (1024,), Hq=8, Hkv=1, kmax=4, selection="fixed2", g=8, W=32),
    2: Workload("8k-community", 2, (8192,), Hq=32, Hkv=8, kmax=16, selection="community",
                communities=8, g=8, W=64),
    3: Workload("32k-community", 3, (32768,), Hq=32, Hkv=8, kmax=32, selection="community",
                communities=16, g=8, W=128),
    4: Workload("64k-community", 4, (65536,), Hq=64, Hkv=8, kmax=32, selection="community",
                communities=32, g=8, W=128),
    5: Workload("ragged-8k16k32k64k-uniform", 5, (8192, 16384, 32768, 65536), Hq=32, Hkv=8,
                kmax=64, selection="uniform", shuffled_pages=True, g=8, W=128),
}


def _gen(wl: Workload, stream: int, head: int = 0, salt: int = 0) -> torch.Generator:
    ss = np.random.SeedSequence([wl.seed_id, stream, head, salt, 0x5057])
    seed = int(ss.generate_state(1, np.uint64)[0] & np.uint64(0x7FFFFFFFFFFFFFFF))
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def cu_seqlens_of(seqlens) -> np.ndarray:
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(seqlens, dtype=np.int64))
    return cu


def pages_of(n_tokens: int) -> int:
    return (n_tokens + PAGE - 1) // PAGE


def _draw_subset(gen, elig: torch.Tensor, m: int) -> torch.Tensor:
    """For each row, up to m distinct column indices drawn uniformly without
    replacement among the True entries of `elig` (random-key sampling).
    Returns int32 [rows, m], -1 where a row had fewer than m eligible columns."""
    rows, cols = elig.shape
    if m <= 0 or cols == 0:
        return torch.full((rows, max(m, 0)), -1, dtype=torch.int32)
    keys = torch.rand(rows, cols, generator=gen)
    keys = torch.where(elig, keys, torch.full_like(keys, 2.0))
    mm = min(m, cols)
    vals, idx = torch.topk(keys, mm, dim=1, largest=False, sorted=True)
    idx = torch.where(vals < 2.0, idx, torch.full_like(idx, -1)).to(torch.int32)
    if mm < m:
        idx = torch.cat([idx, torch.full((rows, m - mm), -1, dtype=torch.int32)], dim=1)
    return idx


def make_selection(wl: Workload, chunk: int = 4096) -> np.ndarray:
    """sel_pages int32 [T, Hkv, kmax] (logical page ids, -1 padded)."""
    T, H, k = wl.T, wl.Hkv, wl.kmax
    sel = torch.full((T, H, k), -1, dtype=torch.int32)
    cu = cu_seqlens_of(wl.seqlens)
    for b, n in enumerate(wl.seqlens):
        P = pages_of(n)
        for h in range(H):
            gsel = _gen(wl, STREAM_SEL, h, salt=b)
            if wl.selection == "community":
                C = wl.communities
                gcomm = _gen(wl, STREAM_COMM, h, salt=b)
                perm = torch.randperm(max(P - 1, 0), generator=gcomm) + 1  # pages 1..P-1
                comm = torch.full((P,), -1, dtype=torch.int64)
                comm[perm] = torch.arange(P - 1, dtype=torch.int64) % C
            for s in range(0, n, chunk):
                e = min(n, s + chunk)
                pos = torch.arange(s, e, dtype=torch.int64)
                o = pos // PAGE
                p = torch.arange(P, dtype=torch.int64)[None, :]
                rows = sel[cu[b] + s: cu[b] + e, h]
                if wl.selection == "fixed2":
                    elig = (p >= 1) & (p < o[:, None])
                    draws = _draw_subset(gsel, elig, k - 2)
                    head = torch.stack([o, torch.zeros_like(o)], 1).to(torch.int32)
                    first = torch.where(o == 0, torch.full_like(o, -1), torch.zeros_like(o))
                    head[:, 1] = first.to(torch.int32)
                    rows[:, :2] = head
                    rows[:, 2:] = draws
                elif wl.selection == "community":
                    blk = pos // wl.block
                    pair = torch.stack([(2 * blk) % C, (2 * blk + 1) % C], 1)
                    c_t = torch.gather(pair, 1, (pos % 2)[:, None])
                    elig = (p >= 1) & (p < o[:, None]) & (comm[None, :] == c_t)
                    draws = _draw_subset(gsel, elig, k - 2)
                    rows[:, 0] = o.to(torch.int32)
                    rows[:, 1] = torch.where(o == 0, torch.full_like(o, -1),
                                             torch.zeros_like(o)).to(torch.int32)
                    rows[:, 2:] = draws
                elif wl.selection == "uniform":
                    elig = p < o[:, None]
                    draws = _draw_subset(gsel, elig, k - 1)
                    rows[:, 0] = o.to(torch.int32)
                    rows[:, 1:] = draws
                else:
                    raise ValueError(f"unknown selection mode {wl.selection!r}")
    return sel.numpy()


def make_page_table(wl: Workload) -> tuple[np.ndarray, int]:
    """page_table int32 [B, max_pages] and the physical pool size."""
    P = [pages_of(n) for n in wl.seqlens]
    maxp = max(P) if P else 0
    total = int(sum(P))
    pt = np.full((wl.B, maxp), -1, dtype=np.int32)
    if wl.shuffled_pages:
        perm = torch.randperm(total, generator=_gen(wl, STREAM_PT)).numpy().astype(np.int32)
    else:
        perm = np.arange(total, dtype=np.int32)
    off = 0
    for b, pb in enumerate(P):
        pt[b, :pb] = perm[off:off + pb]
        off += pb
    return pt, total


def _e4m3_codes(x: torch.Tensor) -> torch.Tensor:
    """float32 -> FP8 E4M3 (round to nearest even, values pre-clipped to +-448) -> uint8 codes."""
    return x.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def make_kv(wl: Workload, page_table: np.ndarray, n_phys: int, chunk_pages: int = 256):
    """K_pages, V_pages uint8 [P_phys, Hkv, 64, 128] filled per logical page, then placed at
    their physical slots.  Entries are E4M3(N(0,1)) codes."""
    shape = (n_phys, wl.Hkv, PAGE, HEAD_DIM)
    out = []
    for stream in (STREAM_K, STREAM_V):
        g = _gen(wl, stream)
        logical = torch.empty(shape, dtype=torch.uint8)
        for s in range(0, n_phys, chunk_pages):
            e = min(n_phys, s + chunk_pages)
            logical[s:e] = _e4m3_codes(torch.randn((e - s,) + shape[1:], generator=g))
        phys = torch.empty_like(logical)
        flat_idx = []
        for b in range(wl.B):
            pb = pages_of(wl.seqlens[b])
            flat_idx.append(page_table[b, :pb])
        idx = torch.from_numpy(np.concatenate(flat_idx).astype(np.int64)) if flat_idx else \
            torch.zeros(0, dtype=torch.int64)
        phys[idx] = logical[: idx.numel()]
        out.append(phys.numpy())
    return out[0], out[1]


def make_q(wl: Workload, chunk_tokens: int = 8192) -> np.ndarray:
    """Q as raw bf16 bits, uint16 [T, Hq, 128]; values bf16(N(0,1))."""
    g = _gen(wl, STREAM_Q)
    q = torch.empty((wl.T, wl.Hq, HEAD_DIM), dtype=torch.bfloat16)
    for s in range(0, wl.T, chunk_tokens):
        e = min(wl.T, s + chunk_tokens)
        q[s:e] = torch.randn((e - s, wl.Hq, HEAD_DIM), generator=g).to(torch.bfloat16)
    return q.view(torch.int16).numpy().view(np.uint16)


def make_inputs(wl: Workload) -> dict:
    """All inputs of one workload as numpy arrays (CPU).  Deterministic per workload."""
    pt, n_phys = make_page_table(wl)
    K, V = make_kv(wl, pt, n_phys)
    return {
        "cu_seqlens": cu_seqlens_of(wl.seqlens),
        "sel_pages": make_selection(wl),
        "Q": make_q(wl),
        "K_pages": K,
        "V_pages": V,
        "page_table": pt,
        "n_phys": n_phys,
        "k_scale": wl.k_scale,
        "v_scale": wl.v_scale,
        "sm_scale": wl.sm_scale,
    }
