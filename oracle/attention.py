"""Block-causal multi-scale attention with per-source-scale probability mass
(the calibration measurement), and pruned-cache attention.

Definitions (fp64 throughout; inputs are the exact bf16 values widened):

* logit   x_ij = tau_h * (q_i . k_j) / sqrt(D) + beta[h][scale(j)]
  The pages give no softmax scale or temperature placement; 1/sqrt(D) is the
  standard scale, the per-head temperature multiplies the scaled dot product
  and the per-(head, source scale) bias is added after it (library reading).
* mask    a query of scale k sees every key of scales 0..k, the whole of its
  own scale included ([Review] Figure 3 caption: rows are the tokens of the
  current scale in raster order, columns the tokens of the scales so far).
* softmax p_ij = exp(x_ij - max_j x_ij) / sum_j exp(x_ij - max_j x_ij);
  O_i = sum_j p_ij v_j.
* mass    m_i(s) = sum over keys j of scale s of p_ij.  [HeatKV] Method
  step 2: attention probabilities are aggregated per layer, head, source
  scale and future scale; M[h][s][k] is the mean of m_i(s) over the B * n_k
  query rows of scale k (seeds folded into the batch), 0 for s > k.
* pruned  a query of scale k of head h attends to the retained past scales
  s < k of that head (ascending order) followed by its own scale k, which is
  always attended ([AMS-KV] Abstract: attending to the local scale matters
  most; [HeatKV] Method step 5: the static schedule is applied at inference).

Parity: the plain definitions above are exact; pinned by tests against closed
forms (uniform attention, bias-only attention), the mass-sums-to-one
invariant, a textbook softmax-attention library routine on a single scale,
and bit-exact equality of pruned attention at a 100% budget with full
attention.
"""
from __future__ import annotations

import math

import numpy as np

from .scales import ScaleGeometry


def attend(q_rows: np.ndarray, keys: np.ndarray, vals: np.ndarray, tau_h: float,
           col_bias: np.ndarray, D: int):
    """Plain softmax attention of some query rows over one key list.

    q_rows [n][D], keys [m][D], vals [m][Dv], col_bias [m] -- all fp64.
    Returns (O [n][Dv], P [n][m])."""
    x = (float(tau_h) * (q_rows @ keys.T)) / math.sqrt(D) + col_bias[None, :]
    x_max = x.max(axis=1, keepdims=True)
    e = np.exp(x - x_max)
    p = e / e.sum(axis=1, keepdims=True)
    return p @ vals, p


def _col_bias(geom: ScaleGeometry, bias_h, key_scales) -> np.ndarray:
    if bias_h is None:
        return np.zeros(len(key_scales), dtype=np.float64)
    b = np.asarray(bias_h, dtype=np.float64)
    return b[np.asarray(key_scales, dtype=np.int64)]


def block_causal_attention(q, k, v, sides, tau, bias=None):
    """Full block-causal attention over a whole [B][H][T][D] stack.

    q, k, v: fp64 arrays [B][H][T][D]; tau [H]; bias [H][S] or None.
    Returns (O [B][H][T][D], mass [B][H][T][S]) where mass[b,h,i,s] = m_i(s)."""
    geom = ScaleGeometry(sides)
    B, H, T, D = q.shape
    assert T == geom.T
    O = np.zeros((B, H, T, v.shape[3]), dtype=np.float64)
    mass = np.zeros((B, H, T, geom.S), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for kk in range(geom.S):
                r0, r1 = geom.off[kk], geom.off[kk] + geom.n[kk]
                Lk = geom.L[kk]
                keys = np.ascontiguousarray(k[b, h, :Lk])
                vals = np.ascontiguousarray(v[b, h, :Lk])
                cb = _col_bias(geom, None if bias is None else bias[h], geom.scale_of[:Lk])
                o, p = attend(np.ascontiguousarray(q[b, h, r0:r1]), keys, vals, tau[h], cb, D)
                O[b, h, r0:r1] = o
                for s in range(kk + 1):
                    mass[b, h, r0:r1, s] = p[:, geom.off[s]:geom.off[s] + geom.n[s]].sum(axis=1)
    return O, mass


def attention_rows(q_rows, k_bh, v_bh, sides, query_scale, tau_h, bias_h=None):
    """Full block-causal attention for some query rows of one (batch, head)
    and one query scale k: keys are k_bh[:L_k].  Returns (O rows, mass rows
    [n][S]).  Used for sampled checks at sizes where the whole stack is too
    slow on the CPU."""
    geom = ScaleGeometry(sides)
    Lk = geom.L[query_scale]
    D = q_rows.shape[1]
    cb = _col_bias(geom, bias_h, geom.scale_of[:Lk])
    o, p = attend(np.ascontiguousarray(q_rows), np.ascontiguousarray(k_bh[:Lk]),
                  np.ascontiguousarray(v_bh[:Lk]), tau_h, cb, D)
    m = np.zeros((q_rows.shape[0], geom.S), dtype=np.float64)
    for s in range(query_scale + 1):
        m[:, s] = p[:, geom.off[s]:geom.off[s] + geom.n[s]].sum(axis=1)
    return o, m


def scas_mass(mass, sides):
    """M[h][s][k] = mean over the B * n_k rows of scale k of m_i(s).

    mass: [B][H][T][S] from block_causal_attention.  Returns [H][S][S] fp64
    indexed [h][s][k]; zero for s > k."""
    geom = ScaleGeometry(sides)
    B, H, T, S = mass.shape
    M = np.zeros((H, S, S), dtype=np.float64)
    for h in range(H):
        for kk in range(S):
            r0, r1 = geom.off[kk], geom.off[kk] + geom.n[kk]
            rows = mass[:, h, r0:r1, :]                     # [B][n_k][S]
            for s in range(kk + 1):
                M[h, s, kk] = rows[:, :, s].sum() / (B * geom.n[kk])
    return M


def pruned_attention(q, k_dense, v_dense, keep_layer, sides, tau, bias=None, query_scale=-1):
    """Pruned-cache attention of one layer.

    q: fp64 [B][H][Tq][D] -- all scales' queries (query_scale = -1, Tq = T) or
    one scale's queries (Tq = n_k).  k_dense, v_dense: fp64 [B][H][T][D], the
    uncompressed cache of this layer.  keep_layer: [H][S] 0/1.
    For head h and query scale k the keys are: for each s < k with
    keep[h][s] = 1 in ascending order, the rows of scale s; then the rows of
    scale k.  Returns O with the shape of q."""
    geom = ScaleGeometry(sides)
    B, H = q.shape[0], q.shape[1]
    D = q.shape[3]
    scales = range(geom.S) if query_scale < 0 else [query_scale]
    O = np.zeros(q.shape[:3] + (v_dense.shape[3],), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for kk in scales:
                key_idx = []
                for s in range(kk):
                    if keep_layer[h][s]:
                        key_idx.extend(range(geom.off[s], geom.off[s] + geom.n[s]))
                key_idx.extend(range(geom.off[kk], geom.off[kk] + geom.n[kk]))
                key_idx = np.asarray(key_idx, dtype=np.int64)
                keys = np.ascontiguousarray(k_dense[b, h][key_idx])
                vals = np.ascontiguousarray(v_dense[b, h][key_idx])
                cb = _col_bias(geom, None if bias is None else bias[h],
                               [geom.scale_of[j] for j in key_idx])
                if query_scale < 0:
                    r0, r1 = geom.off[kk], geom.off[kk] + geom.n[kk]
                else:
                    r0, r1 = 0, geom.n[kk]
                o, _ = attend(np.ascontiguousarray(q[b, h, r0:r1]), keys, vals, tau[h], cb, D)
                O[b, h, r0:r1] = o
    return O


def pruned_attention_rows(q_rows, k_bh, v_bh, keep_h, sides, query_scale, tau_h, bias_h=None):
    """Pruned attention for some query rows of one (batch, head): same key
    list as pruned_attention.  k_bh, v_bh: the dense [T][D] cache rows."""
    geom = ScaleGeometry(sides)
    key_idx = []
    for s in range(query_scale):
        if keep_h[s]:
            key_idx.extend(range(geom.off[s], geom.off[s] + geom.n[s]))
    key_idx.extend(range(geom.off[query_scale], geom.off[query_scale] + geom.n[query_scale]))
    key_idx = np.asarray(key_idx, dtype=np.int64)
    cb = _col_bias(geom, bias_h, [geom.scale_of[j] for j in key_idx])
    o, _ = attend(np.ascontiguousarray(q_rows), np.ascontiguousarray(k_bh[key_idx]),
                  np.ascontiguousarray(v_bh[key_idx]), tau_h, cb, q_rows.shape[1])
    return o
