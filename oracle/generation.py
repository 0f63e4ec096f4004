"""Generation-order application of the static schedule.

[HeatKV] Method step 5: the static schedule keeps cache use within budget as
new scales are generated.  Scale k is generated, its queries attend to the
retained past plus scale k itself (pruned_attention with query_scale = k), and
then scale k's retained blocks are appended to the compacted cache, whose
layout (layout.build_offsets) is final from the start.

[Review] Appendix A, Algorithm 2 CACHESIZEAFTERLAYER(k, l, G_k, G_k-1, E_k):
the body is truncated on the page.  Reading for a static schedule (G_k =
G_k-1 = the dropped pairs, E_k = the entries of scale k): during scale k the
layers run in order, so after layer l the layers 0..l hold their retained
scales <= k and the layers after l their retained scales < k.

Parity: append is exact integer work (pinned: appending every scale in turn
reproduces layout.compact_kv bit for bit); the size accounting is a plain sum,
pinned by the all-kept closed form and its final value = 4 * layer_base[L].
"""
from __future__ import annotations

import numpy as np

from .scales import ScaleGeometry


def append_scale(kc, vc, k_new, v_new, keep, sides, head_off, seg_off, layer_base, scale):
    """Copy scale `scale` of every (layer, batch, head) with keep into kc / vc
    (flat uint16 arrays, modified in place).  k_new, v_new: uint16
    [L][B][H][n_k][D], the new scale's rows."""
    keep = np.asarray(keep)
    L, B, H, nk, D = k_new.shape
    geom = ScaleGeometry(sides)
    assert nk == geom.n[scale]
    for l in range(L):
        R_l = int(layer_base[l + 1] - layer_base[l]) // (B * D)
        for b in range(B):
            for h in range(H):
                if not keep[l, h, scale]:
                    continue
                row = b * R_l + int(head_off[l, h]) + int(seg_off[l, h, scale])
                dst = int(layer_base[l]) + row * D
                kc[dst:dst + nk * D] = k_new[l, b, h].ravel()
                vc[dst:dst + nk * D] = v_new[l, b, h].ravel()


def cache_size_after_layer(keep, sides, B: int, D: int):
    """bytes[k][l] = retained K + V bytes (bf16) held after layer l during the
    generation of scale k: pairs (l', h, s) with keep, and s < k, or s == k and
    l' <= l.  Returns int64 [S][L]."""
    keep = np.asarray(keep)
    L, H, S = keep.shape
    geom = ScaleGeometry(sides)
    out = np.zeros((S, L), dtype=np.int64)
    for k in range(S):
        for l in range(L):
            total = 0
            for lp in range(L):
                for h in range(H):
                    for s in range(S):
                        if keep[lp, h, s] and (s < k or (s == k and lp <= l)):
                            total += geom.n[s] * B * D * 2 * 2
            out[k, l] = total
    return out
