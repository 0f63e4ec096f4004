"""Stability of S-CAS rankings across calibration runs.

[HeatKV] Results: S-CAS rankings remain stable with a small calibration set,
so the schedule can be prepared before inference; [Review] Figure 6 caption:
stability of S-CAS head-scale rankings across calibration runs.  The pages
name no statistic; this library reports, over the candidate pairs
(l, h, s >= n_sinks) of two runs on disjoint seed sets:

* Spearman's rank correlation: the Pearson correlation of the two vectors of
  average ranks (tied values share the mean of their positions);
* the Jaccard overlap of the pairs the two runs' schedules drop at a budget.

Parity: pinned against scipy.stats.spearmanr (an independent library routine)
and the closed forms 1 (identical runs) and -1 (reversed order).
"""
from __future__ import annotations

import numpy as np

from .schedule import build_schedule


def average_ranks(values):
    v = np.asarray(values, dtype=np.float64)
    order = sorted(range(len(v)), key=lambda i: (v[i], i))
    ranks = np.zeros(len(v))
    i = 0
    while i < len(order):
        j = i
        while j + 1 < len(order) and v[order[j + 1]] == v[order[i]]:
            j += 1
        for t in range(i, j + 1):
            ranks[order[t]] = (i + j) / 2.0 + 1.0
        i = j + 1
    return ranks


def rank_stability(scas_a, scas_b, sides, budget_bp: int, n_sinks: int):
    """(spearman, drop_jaccard) of two S-CAS arrays [L][H][S]."""
    a = np.asarray(scas_a, dtype=np.float64)[:, :, n_sinks:].ravel()
    b = np.asarray(scas_b, dtype=np.float64)[:, :, n_sinks:].ravel()
    ra, rb = average_ranks(a), average_ranks(b)
    da, db = ra - ra.mean(), rb - rb.mean()
    den = np.sqrt((da * da).sum() * (db * db).sum())
    spearman = float((da * db).sum() / den) if den > 0 else 0.0
    ka = build_schedule(scas_a, sides, budget_bp, n_sinks)
    kb = build_schedule(scas_b, sides, budget_bp, n_sinks)
    drop_a, drop_b = ka == 0, kb == 0
    union = int((drop_a | drop_b).sum())
    jaccard = float((drop_a & drop_b).sum()) / union if union else 1.0
    return spearman, jaccard
