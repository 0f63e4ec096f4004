"""Time-varying schedule: BINARY-HEATKV with GREEDYEARLYPRUNING.

[Review] Figure 4 caption (Algorithm 1): for each source scale i an order O_i
ranks the (layer, head) squares from least to most dependent on the tokens of
scale i; after scale k, G_k is the union of the length-N_k prefixes of the O_i
(i <= k) and must be absent by the end of scale k.  [HeatKV] Method step 5: a
static schedule and greedy early pruning keep cache use within the budget as
new scales are generated.  The pages leave N_k undefined.  Reading taken:

* O_i: ascending (S-CAS[l][h][i], l, h) over all (layer, head), non-sink i;
* the budget is absolute, budget_bp / 10000 of the final full cache F;
* N_k is the smallest prefix length, non-decreasing in k, such that the cache
  after step k -- the sink scales <= k of every head plus the non-sink scales
  i <= k of the (L*H - N_k) heads outside the prefixes -- fits the budget.

Outputs N_k and, per pair, the first step at which it must be absent (255 if
never).  The retained set after step k is keep_k[l][h][i] = (i <= k and
evict_step[l][h][i] > k).

Parity: pinned by brute force over N (minimality and the budget at every step)
and by the full-budget case (nothing evicted).
"""
from __future__ import annotations

import numpy as np

from .scales import ScaleGeometry
from .schedule import BudgetError


def early_pruning_schedule(scas, sides, budget_bp: int, n_sinks: int):
    scas = np.asarray(scas, dtype=np.float64)
    L, H, S = scas.shape
    geom = ScaleGeometry(sides)
    LH = L * H
    F = LH * geom.T
    if LH * sum(geom.n[:n_sinks]) * 10000 > budget_bp * F:
        raise BudgetError("sink scales alone exceed the budget")
    rank = np.zeros((S, LH), dtype=np.int64)
    for i in range(n_sinks, S):
        order = sorted(range(LH), key=lambda lh: (scas.reshape(LH, S)[lh, i], lh))
        for pos, lh in enumerate(order):
            rank[i, lh] = pos
    prefix = np.zeros(S, dtype=np.int32)
    N = 0
    for k in range(S):
        nonsink = sum(geom.n[i] for i in range(n_sinks, k + 1))
        sinks_k = LH * sum(geom.n[i] for i in range(min(n_sinks, k + 1)))
        while N < LH and (sinks_k + (LH - N) * nonsink) * 10000 > budget_bp * F:
            N += 1
        prefix[k] = N if nonsink > 0 else 0
    evict = np.full((L, H, S), 255, dtype=np.uint8)
    for lh in range(LH):
        l, h = divmod(lh, H)
        for i in range(n_sinks, S):
            for k in range(i, S):
                if rank[i, lh] < prefix[k]:
                    evict[l, h, i] = k
                    break
    return prefix, evict


def keep_after_step(evict, k: int):
    """Retained pairs after step k: scale i <= k not yet evicted."""
    evict = np.asarray(evict)
    S = evict.shape[2]
    idx = np.arange(S)[None, None, :]
    return ((idx <= k) & (evict.astype(np.int64) > k)).astype(np.uint8)
