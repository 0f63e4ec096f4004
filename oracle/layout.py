"""Offset tables and compaction of the retained scale blocks into a per-head
ragged K/V layout.

The pages fix no memory layout ([HeatKV] Method step 5 only says the static
schedule is applied during inference, head-specific per the Abstract); this
is the library's layout, stated once in its C header and restated here:

  R[l][h]        = sum_s keep[l][h][s] * n_s            rows kept by head h
  R_l            = sum_h R[l][h]                        rows per batch element
  head_off[l][h] = sum_{h' < h} R[l][h']
  seg_off[l][h][s] = sum_{s' < s} keep[l][h][s'] * n_s'  if keep, else -1
  past_len[l][h][k] = sum_{s < k} keep[l][h][s] * n_s
  layer_base[l]  = sum_{l' < l} B * R_l' * D            (elements; L+1 entries)

Layer l's compacted K (and V) is a [B][R_l][D] block starting at element
layer_base[l]; token t of kept scale s of (b, h) sits at row
b * R_l + head_off[l][h] + seg_off[l][h][s] + t.  Within a head the kept
scales are ascending, raster order inside each scale.

Parity: exact integer work; pinned by closed-form prefix sums (all kept ->
head_off = h*T, seg_off = off_s, ...) and by identity-coded compaction.
"""
from __future__ import annotations

import numpy as np

from .scales import ScaleGeometry


def build_offsets(keep, sides, B: int, D: int):
    """Returns (head_off int32 [L][H], seg_off int32 [L][H][S],
    past_len int32 [L][H][S], layer_base int64 [L+1])."""
    keep = np.asarray(keep)
    L, H, S = keep.shape
    geom = ScaleGeometry(sides)
    head_off = np.zeros((L, H), dtype=np.int32)
    seg_off = np.full((L, H, S), -1, dtype=np.int32)
    past_len = np.zeros((L, H, S), dtype=np.int32)
    layer_base = np.zeros(L + 1, dtype=np.int64)
    for l in range(L):
        rows_before_head = 0
        for h in range(H):
            head_off[l, h] = rows_before_head
            running = 0
            for s in range(S):
                past_len[l, h, s] = running
                if keep[l, h, s]:
                    seg_off[l, h, s] = running
                    running += geom.n[s]
            rows_before_head += running
        layer_base[l + 1] = layer_base[l] + B * rows_before_head * D
    return head_off, seg_off, past_len, layer_base


def compact_kv(k_dense, v_dense, keep, sides, head_off, seg_off, layer_base):
    """Gather retained scale blocks.

    k_dense, v_dense: uint16 (raw bf16 bits) [L][B][H][T][D].  Returns flat
    uint16 arrays kc, vc of length layer_base[L]."""
    keep = np.asarray(keep)
    L, B, H, T, D = k_dense.shape
    geom = ScaleGeometry(sides)
    total = int(layer_base[L])
    kc = np.zeros(total, dtype=k_dense.dtype)
    vc = np.zeros(total, dtype=v_dense.dtype)
    for l in range(L):
        R_l = int(layer_base[l + 1] - layer_base[l]) // (B * D)
        for b in range(B):
            for h in range(H):
                for s in range(geom.S):
                    if not keep[l, h, s]:
                        continue
                    row = b * R_l + int(head_off[l, h]) + int(seg_off[l, h, s])
                    dst = int(layer_base[l]) + row * D
                    n = geom.n[s] * D
                    src_k = k_dense[l, b, h, geom.off[s]:geom.off[s] + geom.n[s]].ravel()
                    src_v = v_dense[l, b, h, geom.off[s]:geom.off[s] + geom.n[s]].ravel()
                    kc[dst:dst + n] = src_k
                    vc[dst:dst + n] = src_v
    return kc, vc
