"""Helpers for the GPU tests: moving generator bits to and from the device and
driving the library's calls for one workload.  Marshalling only -- no step of
the method is computed here."""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_compression_cas_b200 as vark


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def status_word() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def check_status(st: torch.Tensor):
    torch.cuda.synchronize()
    assert int(st.item()) == 0, vark.vark_status_string(int(st.item()))


class Tables:
    """Device offset tables of a keep schedule."""

    def __init__(self, keep: np.ndarray, sides, B: int, D: int):
        L, H, S = keep.shape
        self.keep_host = np.ascontiguousarray(keep, dtype=np.uint8)
        self.keep = torch.from_numpy(self.keep_host).cuda()
        self.head_off = torch.empty((L, H), dtype=torch.int32, device="cuda")
        self.seg_off = torch.empty((L, H, S), dtype=torch.int32, device="cuda")
        self.past_len = torch.empty((L, H, S), dtype=torch.int32, device="cuda")
        self.layer_base = torch.empty(L + 1, dtype=torch.int64, device="cuda")
        vark.vark_build_offsets(self.keep, sides, B, D, self.head_off, self.seg_off, self.past_len, self.layer_base)
        # rows per batch element of each layer, read back from layer_base
        self.base_host = self.layer_base.cpu().numpy()
        self.R_l = np.diff(self.base_host) // (B * D)
        self.total = int(self.base_host[-1])
        self.L, self.H, self.S, self.B, self.D = L, H, S, B, D

    def kc_rows(self, l: int) -> int:
        return int(self.R_l[l]) * self.B

    def elem_base(self, l: int) -> int:
        return int(self.base_host[l])


def compact(k_dense: torch.Tensor, v_dense: torch.Tensor, tab: Tables, sides):
    """k_dense/v_dense: [L][B][H][T][D] bf16.  Returns flat kc, vc."""
    L, B, H, T, D = k_dense.shape
    kc = torch.empty(max(tab.total, 8), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty(max(tab.total, 8), dtype=torch.bfloat16, device="cuda")
    vark.vark_compact_kv(k_dense, v_dense, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off,
                         tab.layer_base, kc, vc)
    return kc, vc


def pruned_layer(q, kc, vc, k_dense_l, v_dense_l, tab: Tables, l: int, sides, query_scale, tau, bias):
    """Pruned attention of layer l.  q: [B][H][Tq][D]; k_dense_l: [B][H][T][D]."""
    out = torch.empty_like(q)
    st = status_word()
    base = tab.elem_base(l)
    rows = tab.kc_rows(l)
    D = q.shape[3]
    kcl = kc[base:base + rows * D] if rows > 0 else None
    vcl = vc[base:base + rows * D] if rows > 0 else None
    vark.vark_pruned_attention(q, kcl, vcl, rows, k_dense_l, v_dense_l, sides, query_scale, tab.head_off[l],
                               tab.seg_off[l], tab.past_len[l], tau, bias, out, st)
    check_status(st)
    return out
