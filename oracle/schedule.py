"""S-CAS and the static keep[layer][head][scale] schedule.

* S-CAS.  [HeatKV] Abstract and Method step 3: the Scale-dependent Cumulative
  Attention Score ranks how strongly each head depends on each earlier scale,
  from attention aggregated per (layer, head, source scale, future scale)
  (Method step 2).  The pages print no formula; this library defines
    S-CAS[l][h][s] = sum over k > s of M[l][h][s][k]
  with M the mean over scale-k queries of the mass on scale-s keys (see
  attention.scas_mass), averaged over calibration seeds.  The last scale
  therefore scores 0.  Parity against the paper's own S-CAS values: parity
  unpinned (the pages print none); the sum itself is pinned by closed forms.

* Schedule.  [HeatKV] Method step 4: the memory budget decides how many
  low-ranked head-scale pairs are removed while the early sink scales are
  retained; Abstract: one static schedule for a chosen budget.  Readings:
  - the full cache F counts every (layer, head, scale) at the end of
    generation, in tokens (bytes = tokens * D * 2 * 2 for every pair, so the
    token count decides the budget exactly); [HeatKV] Table 1 states budgets
    as fractions of the full cache;
  - candidates are every (l, h, s) with s >= n_sinks, ranked by ascending
    (S-CAS, l, h, s) -- ties broken by index;
  - pairs are dropped in that order and the walk stops at the first point
    where kept * 10000 <= budget_bp * F (no skipping; equality meets it);
  - if the sinks alone exceed the budget there is no schedule (BudgetError);
  - the local scale of a query is attended from the dense cache at
    inference, so it is not a greedy exception.
  Parity: pinned by brute force over every drop set on <= 8 candidates and
  by the all-kept / index-order special cases.
"""
from __future__ import annotations

import numpy as np

from .scales import ScaleGeometry


class BudgetError(ValueError):
    """The sink scales alone exceed the requested budget."""


def scas_from_mass(M, n_calls: int = 1):
    """S-CAS[l][h][s] = (1/n_calls) * sum_{k > s} M[l][h][s][k].

    M: [L][H][S][S] (or [H][S][S]) accumulated over n_calls calibration calls,
    each adding the mean over its own B * n_k rows."""
    M = np.asarray(M, dtype=np.float64)
    squeeze = M.ndim == 3
    if squeeze:
        M = M[None]
    L, H, S, _ = M.shape
    out = np.zeros((L, H, S), dtype=np.float64)
    for l in range(L):
        for h in range(H):
            for s in range(S):
                acc = 0.0
                for k in range(s + 1, S):
                    acc += M[l, h, s, k]
                out[l, h, s] = acc / n_calls
    return out[0] if squeeze else out


def full_cache_tokens(L: int, H: int, sides) -> int:
    return L * H * ScaleGeometry(sides).T


def build_schedule(scas, sides, budget_bp: int, n_sinks: int) -> np.ndarray:
    """Greedy global drop of the lowest-S-CAS head-scale pairs.

    scas: fp64 [L][H][S].  Returns keep uint8 [L][H][S]."""
    scas = np.asarray(scas, dtype=np.float64)
    L, H, S = scas.shape
    geom = ScaleGeometry(sides)
    assert S == geom.S
    F = full_cache_tokens(L, H, sides)
    keep = np.ones((L, H, S), dtype=np.uint8)
    kept = F
    if kept * 10000 <= budget_bp * F:
        return keep
    sink_tokens = L * H * sum(geom.n[:n_sinks])
    if sink_tokens * 10000 > budget_bp * F:
        raise BudgetError("sink scales alone exceed the budget")
    candidates = []
    for l in range(L):
        for h in range(H):
            for s in range(n_sinks, S):
                candidates.append((float(scas[l, h, s]), l, h, s))
    candidates.sort()
    for _, l, h, s in candidates:
        keep[l, h, s] = 0
        kept -= geom.n[s]
        if kept * 10000 <= budget_bp * F:
            break
    return keep
