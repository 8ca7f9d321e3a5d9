"""Python binding of the PageWeaver hot path (argument marshalling only).

Every step of the path runs in libpw.so's kernels; torch supplies device memory and streams.
Names follow the C ABI (include/pw.h): pw_groups_size, pw_group, pw_attn.  `prefill` runs one
complete call (pw_group then pw_attn on the current stream).
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib
from ._lib import PwError, PwGroups


def _ptr(t: torch.Tensor | None):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def _stream(stream) -> C.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _host_cu(cu_host) -> np.ndarray:
    if isinstance(cu_host, torch.Tensor):
        cu_host = cu_host.detach().cpu().numpy()
    return np.ascontiguousarray(cu_host, dtype=np.int32)


def _check(code: int, where: str):
    if code != _lib.PW_OK:
        raise PwError(code, where)


def pw_groups_size(cu_seqlens_host, Hkv: int, kmax: int, W: int, g: int):
    """(n_groups, union_cap, words, workspace_bytes) for these shapes (host only)."""
    L = _lib.load()
    cu = _host_cu(cu_seqlens_host)
    ng, uc, wd, ws = C.c_int64(), C.c_int64(), C.c_int32(), C.c_size_t()
    _check(L.pw_groups_size(cu.ctypes.data_as(C.c_void_p), len(cu) - 1, Hkv, kmax, W, g,
                            C.byref(ng), C.byref(uc), C.byref(wd), C.byref(ws)), "pw_groups_size")
    return ng.value, uc.value, wd.value, ws.value


@dataclass
class Groups:
    """Device buffers of struct pw_groups (see include/pw.h for their layouts)."""
    qids: torch.Tensor
    gsize: torch.Tensor
    gmeta: torch.Tensor
    union_off: torch.Tensor
    union_pages: torch.Tensor
    bits: torch.Tensor
    sched: torch.Tensor
    workspace: torch.Tensor
    n_groups: int
    union_cap: int
    words: int
    g: int
    W: int

    @classmethod
    def allocate(cls, T: int, Hkv: int, cu_seqlens_host, kmax: int, W: int, g: int,
                 device="cuda") -> "Groups":
        ng, uc, words, ws = pw_groups_size(cu_seqlens_host, Hkv, kmax, W, g)
        i32 = dict(dtype=torch.int32, device=device)
        return cls(
            qids=torch.empty(max(ng * g, 1), **i32),
            gsize=torch.empty(max(ng, 1), **i32),
            gmeta=torch.empty(max(ng * 3, 1), **i32),
            union_off=torch.empty(ng + 1, **i32),
            union_pages=torch.empty(max(uc, 1), **i32),
            bits=torch.empty(max(T * Hkv * words, 1), dtype=torch.int32, device=device),
            sched=torch.zeros(1, **i32),
            workspace=torch.empty(ws, dtype=torch.uint8, device=device),
            n_groups=ng, union_cap=uc, words=words, g=g, W=W)

    def struct(self) -> PwGroups:
        return PwGroups(self.qids.data_ptr(), self.gsize.data_ptr(), self.gmeta.data_ptr(),
                        self.union_off.data_ptr(), self.union_pages.data_ptr(),
                        self.bits.data_ptr(), self.sched.data_ptr(), self.n_groups,
                        self.union_cap, self.words, self.g)

    def to_host(self) -> dict:
        """Group arrays copied to the host, trimmed to n_groups and the union length."""
        n, g = self.n_groups, self.g
        uo = self.union_off.cpu().numpy()
        return {
            "n_groups": n,
            "g": g,
            "qids": self.qids[: n * g].cpu().numpy().reshape(n, g),
            "gsize": self.gsize[:n].cpu().numpy(),
            "gmeta": self.gmeta[: 3 * n].cpu().numpy().reshape(n, 3),
            "union_off": uo,
            "union_pages": self.union_pages[: int(uo[n])].cpu().numpy() if n > 0 else
            np.zeros(0, np.int32),
        }


def new_status(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(status: torch.Tensor, where: str = "device"):
    """Read the device status word (synchronises) and raise on an error."""
    _check(int(status.item()), where)


def pw_group(sel_pages: torch.Tensor, cu_seqlens: torch.Tensor, cu_seqlens_host, W: int, g: int,
             groups: Groups | None = None, status: torch.Tensor | None = None,
             stream=None) -> Groups:
    """Bounded-window greedy grouping on the GPU (include/pw.h, pw_group)."""
    L = _lib.load()
    assert sel_pages.is_cuda and sel_pages.dtype == torch.int32 and sel_pages.is_contiguous()
    assert cu_seqlens.is_cuda and cu_seqlens.dtype == torch.int32
    T, Hkv, kmax = sel_pages.shape
    cu = _host_cu(cu_seqlens_host)
    if groups is None:
        groups = Groups.allocate(T, Hkv, cu, kmax, W, g, device=sel_pages.device)
    if status is None:
        status = new_status(sel_pages.device)
    st = groups.struct()
    _check(L.pw_group(_ptr(sel_pages), _ptr(cu_seqlens), cu.ctypes.data_as(C.c_void_p),
                      len(cu) - 1, Hkv, kmax, W, g, C.byref(st), _ptr(groups.workspace),
                      groups.workspace.numel(), _ptr(status), _stream(stream)), "pw_group")
    return groups


def pw_attn(Q: torch.Tensor, K_pages: torch.Tensor, V_pages: torch.Tensor,
            page_table: torch.Tensor, cu_seqlens: torch.Tensor, groups: Groups,
            k_scale: float = 1.0, v_scale: float = 1.0, sm_scale: float | None = None,
            O: torch.Tensor | None = None, status: torch.Tensor | None = None,
            stream=None, cu_seqlens_host=None) -> torch.Tensor:
    """ID-aware union attention (include/pw.h, pw_attn).  Q bf16 [T, Hq, 128];
    K_pages/V_pages uint8 E4M3 codes [n_phys, Hkv, 64, 128]; page_table int32 [B, max_pages]
    with B = len(cu_seqlens) - 1; returns O bf16 [T, Hq, 128].  With cu_seqlens_host (a host
    copy of cu_seqlens) the page table's width is checked against the longest sequence."""
    L = _lib.load()
    T, Hq, D = Q.shape
    assert Q.is_cuda and Q.dtype == torch.bfloat16 and Q.is_contiguous() and D == 128
    for t in (K_pages, V_pages, page_table, cu_seqlens):
        assert t.is_cuda and t.device == Q.device and t.is_contiguous()
    assert K_pages.dtype == torch.uint8 and V_pages.dtype == torch.uint8
    assert K_pages.dim() == 4 and tuple(K_pages.shape[2:]) == (64, 128)
    assert K_pages.shape == V_pages.shape
    n_phys, Hkv = K_pages.shape[0], K_pages.shape[1]
    assert Hq % Hkv == 0
    assert cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1
    B = cu_seqlens.numel() - 1
    assert page_table.dtype == torch.int32 and page_table.dim() == 2 and page_table.shape[0] == B
    assert groups.bits.numel() >= T * Hkv * groups.words
    if cu_seqlens_host is not None:
        cu = _host_cu(cu_seqlens_host)
        assert len(cu) == B + 1 and int(cu[-1]) == T
        max_len = int(np.max(np.diff(cu))) if B > 0 else 0
        assert page_table.shape[1] >= (max_len + 63) // 64, "page table narrower than a sequence"
    if sm_scale is None:
        sm_scale = 1.0 / float(np.sqrt(D))
    if O is None:
        O = torch.empty_like(Q)
    if status is None:
        status = new_status(Q.device)
    st = groups.struct()
    _check(L.pw_attn(_ptr(Q), _ptr(K_pages), _ptr(V_pages), _ptr(page_table),
                     page_table.shape[1], n_phys, _ptr(cu_seqlens), B, T, Hq,
                     Hkv, float(k_scale), float(v_scale), float(sm_scale), C.byref(st), _ptr(O),
                     _ptr(status), _stream(stream)), "pw_attn")
    return O


def prefill(Q, K_pages, V_pages, page_table, sel_pages, cu_seqlens, cu_seqlens_host, W: int,
            g: int = 8, k_scale: float = 1.0, v_scale: float = 1.0, sm_scale=None,
            groups: Groups | None = None, O=None, status=None, stream=None):
    """One complete call: pw_group then pw_attn on the same stream.  Returns (O, groups)."""
    if status is None:
        status = new_status(Q.device)
    groups = pw_group(sel_pages, cu_seqlens, cu_seqlens_host, W, g, groups=groups, status=status,
                      stream=stream)
    O = pw_attn(Q, K_pages, V_pages, page_table, cu_seqlens, groups, k_scale, v_scale, sm_scale,
                O=O, status=status, stream=stream, cu_seqlens_host=cu_seqlens_host)
    return O, groups


def device_inputs(inp: dict, device="cuda") -> dict:
    """Move a synth.make_inputs() dict to the device with the dtypes the calls expect."""
    return {
        "Q": torch.from_numpy(inp["Q"].view(np.int16)).view(torch.bfloat16).to(device),
        "K_pages": torch.from_numpy(inp["K_pages"]).to(device),
        "V_pages": torch.from_numpy(inp["V_pages"]).to(device),
        "page_table": torch.from_numpy(inp["page_table"]).to(device),
        "sel_pages": torch.from_numpy(inp["sel_pages"]).to(device),
        "cu_seqlens": torch.from_numpy(inp["cu_seqlens"]).to(device),
        "cu_seqlens_host": np.ascontiguousarray(inp["cu_seqlens"], np.int32),
        "k_scale": inp["k_scale"], "v_scale": inp["v_scale"], "sm_scale": inp["sm_scale"],
    }
