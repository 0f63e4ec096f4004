"""Pins of the fp64 oracle against things other than itself: closed forms,
invariants, an independent library routine (torch's scaled-dot-product
attention in fp64 with an explicit block-causal mask), brute force over drop
sets, and planted mistakes that must trip at least one pin."""
from fractions import Fraction
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt
from synth import SIDES_TINY, bf16_bits_to_f32, normal_bf16_bits, derive_key, gen_tau, gen_bias

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _qkv(B, H, T, D, tag=0):
    out = []
    for which in range(3):
        bits = normal_bf16_bits(derive_key(99, tag, which), (B, H, T, D))
        out.append(bf16_bits_to_f32(bits).astype(np.float64))
    return out


def _geom(sides):
    return oracle.ScaleGeometry(sides)


# ---------------------------------------------------------------- attention

def test_mass_rows_sum_to_one_and_scas_column_sums():
    """Every softmax row sums to 1, so sum_{s<=k} M[h][s][k] = 1 per scale."""
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, v = _qkv(2, 3, g.T, 64)
    tau = gen_tau(1, 3).astype(np.float64)
    bias = gen_bias(1, 3, g.S).astype(np.float64)
    _, mass = oracle.block_causal_attention(q, k, v, sides, tau, bias)
    np.testing.assert_allclose(mass.sum(axis=3), 1.0, atol=1e-12, rtol=0)
    M = oracle.scas_mass(mass, sides)
    for kk in range(g.S):
        np.testing.assert_allclose(M[:, :kk + 1, kk].sum(axis=1), 1.0, atol=1e-12, rtol=0)
        assert np.all(M[:, kk + 1:, kk] == 0.0)


def _read_uniform_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "uniform_scas_tiny.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            s, expr = line.split()
            total = Fraction(0)
            for term in expr.split("+"):
                total += Fraction(term)
            vals[int(s)] = total
    return vals


def test_uniform_attention_closed_form_golden():
    """Q = 0, no bias: M[s][k] = n_s / L_k and S-CAS from the golden fixture."""
    sides = SIDES_TINY
    g = _geom(sides)
    _, k, v = _qkv(2, 2, g.T, 64, tag=1)
    q = np.zeros_like(k)
    tau = np.array([0.7, 1.9])
    _, mass = oracle.block_causal_attention(q, k, v, sides, tau, None)
    M = oracle.scas_mass(mass, sides)
    for kk in range(g.S):
        for s in range(kk + 1):
            assert abs(M[0, s, kk] - g.n[s] / g.L[kk]) < 1e-14
    scas = oracle.scas_from_mass(M[None])[0]
    gold = _read_uniform_golden()
    for s, val in gold.items():
        np.testing.assert_allclose(scas[:, s], float(val), atol=1e-14, rtol=0)
    # the golden file's first row written out as the project-page example
    assert abs(float(gold[0]) - (1/5 + 1/14 + 1/30 + 1/55 + 1/91 + 1/155)) < 1e-15


def test_bias_only_closed_form():
    """Q = 0 with a per-scale logit bias: M[s][k] = n_s e^b_s / sum_{s'<=k} n_s' e^b_s'."""
    sides = SIDES_TINY
    g = _geom(sides)
    _, k, v = _qkv(1, 2, g.T, 64, tag=2)
    q = np.zeros_like(k)
    bias = np.array([[0.3, 1.7, 0.0, 2.0, 0.5, 0.0, 1.1], [0, 0, 1.5, 0, 0, 0, 0.2]])
    _, mass = oracle.block_causal_attention(q, k, v, sides, np.array([1.0, 1.3]), bias)
    M = oracle.scas_mass(mass, sides)
    for h in range(2):
        for kk in range(g.S):
            den = sum(g.n[s] * math.exp(bias[h][s]) for s in range(kk + 1))
            for s in range(kk + 1):
                assert abs(M[h, s, kk] - g.n[s] * math.exp(bias[h][s]) / den) < 1e-13


def test_scale_indicator_values_reproduce_mass():
    """V columns set to scale indicators: O[:, s] equals the row mass m_i(s)."""
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, _ = _qkv(1, 2, g.T, 64, tag=3)
    v = np.zeros((1, 2, g.T, g.S))
    for j in range(g.T):
        v[0, :, j, g.scale_of[j]] = 1.0
    O, mass = oracle.block_causal_attention(q, k, v, sides, np.array([1.5, 0.6]),
                                            gen_bias(3, 2, g.S).astype(np.float64))
    np.testing.assert_allclose(O, mass, atol=1e-13, rtol=0)


def _sdpa_reference(q, k, v, allowed, tau, bias_cols):
    """torch fp64 scaled_dot_product_attention with a float mask: bias where
    allowed, -inf elsewhere; scale tau/sqrt(D)."""
    D = q.shape[-1]
    qt = torch.from_numpy(q)[None]
    kt = torch.from_numpy(k)[None]
    vt = torch.from_numpy(v)[None]
    mask = torch.full(allowed.shape, float("-inf"), dtype=torch.float64)
    mask[torch.from_numpy(allowed)] = 0.0
    mask = mask + torch.from_numpy(bias_cols)[None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask[None],
                                                         scale=float(tau) / math.sqrt(D))
    return o[0].numpy()


def test_block_causal_matches_library_attention_with_mask():
    """Whole block-causal stack vs torch SDPA with an explicit scale mask."""
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, v = _qkv(1, 2, g.T, 64, tag=4)
    tau = np.array([0.55, 1.8])
    bias = gen_bias(4, 2, g.S).astype(np.float64)
    O, _ = oracle.block_causal_attention(q, k, v, sides, tau, bias)
    sc = np.array(g.scale_of)
    allowed = sc[None, :] <= sc[:, None]
    for h in range(2):
        ref = _sdpa_reference(q[0, h], k[0, h], v[0, h], allowed, tau[h], bias[h][sc])
        np.testing.assert_allclose(O[0, h], ref, atol=1e-12, rtol=0)


def test_single_scale_is_textbook_attention():
    sides = (5,)
    q, k, v = _qkv(1, 1, 25, 32, tag=5)
    O, mass = oracle.block_causal_attention(q, k, v, sides, np.array([1.25]), None)
    ref = _sdpa_reference(q[0, 0], k[0, 0], v[0, 0], np.ones((25, 25), bool), 1.25, np.zeros(25))
    np.testing.assert_allclose(O[0, 0], ref, atol=1e-13, rtol=0)
    np.testing.assert_allclose(mass[..., 0], 1.0, atol=1e-14)


def test_pruned_at_full_budget_is_full_attention_bit_exact():
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, v = _qkv(2, 2, g.T, 64, tag=6)
    tau = np.array([0.9, 1.4])
    bias = gen_bias(6, 2, g.S).astype(np.float64)
    O_full, _ = oracle.block_causal_attention(q, k, v, sides, tau, bias)
    keep = np.ones((2, g.S), dtype=np.uint8)
    O_pr = oracle.pruned_attention(q, k, v, keep, sides, tau, bias)
    assert np.array_equal(O_full, O_pr)


def test_pruned_matches_library_attention_with_keep_mask():
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, v = _qkv(1, 3, g.T, 64, tag=7)
    tau = np.array([0.9, 1.4, 0.6])
    bias = gen_bias(7, 3, g.S).astype(np.float64)
    rng = np.random.default_rng(7)
    keep = rng.integers(0, 2, size=(3, g.S)).astype(np.uint8)
    keep[:, :2] = 1
    O = oracle.pruned_attention(q, k, v, keep, sides, tau, bias)
    sc = np.array(g.scale_of)
    for h in range(3):
        allowed = ((sc[None, :] < sc[:, None]) & (keep[h][sc][None, :] == 1)) | (sc[None, :] == sc[:, None])
        ref = _sdpa_reference(q[0, h], k[0, h], v[0, h], allowed, tau[h], bias[h][sc])
        np.testing.assert_allclose(O[0, h], ref, atol=1e-12, rtol=0)
    # single-query-scale form gives the same rows
    kq = 5
    O5 = oracle.pruned_attention(q[:, :, g.off[kq]:g.off[kq] + g.n[kq]], k, v, keep, sides, tau, bias, query_scale=kq)
    np.testing.assert_array_equal(O5, O[:, :, g.off[kq]:g.off[kq] + g.n[kq]])


def test_constant_values_give_constant_output():
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, _ = _qkv(1, 2, g.T, 64, tag=8)
    v = np.full((1, 2, g.T, 64), 0.375)
    O, _ = oracle.block_causal_attention(q, k, v, sides, np.array([1.0, 2.0]), None)
    np.testing.assert_allclose(O, 0.375, atol=1e-14, rtol=0)
    keep = np.zeros((2, g.S), dtype=np.uint8)
    O2 = oracle.pruned_attention(q, k, v, keep, sides, np.array([1.0, 2.0]))
    np.testing.assert_allclose(O2, 0.375, atol=1e-14, rtol=0)


def test_row_helpers_agree_with_whole_stack():
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, v = _qkv(1, 2, g.T, 64, tag=9)
    tau = np.array([0.8, 1.1])
    bias = gen_bias(9, 2, g.S).astype(np.float64)
    O, mass = oracle.block_causal_attention(q, k, v, sides, tau, bias)
    kk = 6
    r0, r1 = g.off[kk], g.L[kk]
    o, m = oracle.attention_rows(q[0, 1, r0:r1], k[0, 1], v[0, 1], sides, kk, tau[1], bias[1])
    np.testing.assert_array_equal(o, O[0, 1, r0:r1])
    np.testing.assert_array_equal(m, mass[0, 1, r0:r1])
    keep = np.array([1, 1, 0, 1, 0, 0, 1], dtype=np.uint8)
    Op = oracle.pruned_attention(q, k, v, np.stack([keep, keep]), sides, tau, bias)
    o2 = oatt.pruned_attention_rows(q[0, 0, r0:r1], k[0, 0], v[0, 0], keep, sides, kk, tau[0], bias[0])
    np.testing.assert_array_equal(o2, Op[0, 0, r0:r1])


# ---------------------------------------------------------------- schedule

def _brute_force_drop_set(scores, sizes, budget_bp, F, base_kept):
    """Smallest rank-closed feasible drop set, by enumeration of all subsets.
    Rank-closed: every candidate ranked below a dropped one is dropped too,
    ranks compared pairwise on (score, index)."""
    n = len(scores)
    keys = [(scores[i], i) for i in range(n)]
    best = None
    for mask in range(1 << n):
        X = [i for i in range(n) if mask >> i & 1]
        closed = all(keys[y] > keys[x] for x in X for y in range(n) if not (mask >> y & 1))
        if not closed:
            continue
        kept = base_kept - sum(sizes[i] for i in X)
        if kept * 10000 > budget_bp * F:
            continue
        if best is None or len(X) < len(best):
            best = X
    return best


@pytest.mark.parametrize("trial", range(6))
def test_schedule_matches_brute_force_on_eight_pairs(trial):
    sides = (1, 2, 3, 4, 5, 6)          # 4 candidates per head with sinks 0-1
    g = _geom(sides)
    L, H, n_sinks = 1, 2, 2
    rng = np.random.default_rng(100 + trial)
    scas = rng.uniform(0, 1, size=(L, H, g.S))
    if trial % 2:
        scas = np.round(scas, 1)            # force ties -> index tie-break
    cand = [(l, h, s) for l in range(L) for h in range(H) for s in range(n_sinks, g.S)]
    assert len(cand) == 8
    F = L * H * g.T
    for budget in range(0, 10001, 250):
        sink = L * H * sum(g.n[:n_sinks])
        if sink * 10000 > budget * F:
            with pytest.raises(oracle.BudgetError):
                oracle.build_schedule(scas, sides, budget, n_sinks)
            continue
        keep = oracle.build_schedule(scas, sides, budget, n_sinks)
        dropped = [i for i, (l, h, s) in enumerate(cand) if keep[l, h, s] == 0]
        # the ranking key uses the position in index order as the tie-break
        bf = _brute_force_drop_set([scas[c] for c in cand], [g.n[c[2]] for c in cand], budget, F, F)
        assert sorted(dropped) == sorted(bf), (budget, dropped, bf)
        assert np.all(keep[:, :, :n_sinks] == 1)
        kept = int((keep * np.array(g.n)[None, None, :]).sum())
        assert kept * 10000 <= budget * F


def test_schedule_special_cases():
    sides = SIDES_TINY
    g = _geom(sides)
    scas = np.random.default_rng(0).uniform(size=(2, 3, g.S))
    assert np.all(oracle.build_schedule(scas, sides, 10000, 2) == 1)
    # all-zero S-CAS: drop order is plain index order (l, h, s)
    keep = oracle.build_schedule(np.zeros((2, 3, g.S)), sides, 9000, 2)
    F = 2 * 3 * g.T
    order = [(l, h, s) for l in range(2) for h in range(3) for s in range(2, g.S)]
    kept, ndrop = F, 0
    while kept * 10000 > 9000 * F:
        kept -= g.n[order[ndrop][2]]
        ndrop += 1
    for i, (l, h, s) in enumerate(order):
        assert keep[l, h, s] == (0 if i < ndrop else 1)
    with pytest.raises(oracle.BudgetError):
        oracle.build_schedule(scas, sides, 10, 2)       # 0.1% < sinks (5/155)
    # the last scale scores 0 and is dropped first
    scas2 = np.random.default_rng(1).uniform(0.1, 1, size=(1, 2, g.S))
    scas2[:, :, -1] = 0.0
    keep2 = oracle.build_schedule(scas2, sides, 7000, 2)
    assert np.all(keep2[0, :, -1] == 0)


# ---------------------------------------------------------------- layout

def test_offsets_closed_form_all_kept():
    sides = SIDES_TINY
    g = _geom(sides)
    L, H, B, D = 3, 4, 2, 64
    keep = np.ones((L, H, g.S), dtype=np.uint8)
    head_off, seg_off, past_len, layer_base = oracle.build_offsets(keep, sides, B, D)
    for l in range(L):
        for h in range(H):
            assert head_off[l, h] == h * g.T
            for s in range(g.S):
                assert seg_off[l, h, s] == g.off[s]
                assert past_len[l, h, s] == g.off[s]
    assert list(layer_base) == [l * B * H * g.T * D for l in range(L + 1)]


def test_offsets_invariants_random_keep():
    sides = SIDES_TINY
    g = _geom(sides)
    L, H, B, D = 2, 5, 3, 64
    keep = np.random.default_rng(5).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    head_off, seg_off, past_len, layer_base = oracle.build_offsets(keep, sides, B, D)
    for l in range(L):
        R = [sum(g.n[s] for s in range(g.S) if keep[l, h, s]) for h in range(H)]
        assert list(head_off[l]) == [sum(R[:h]) for h in range(H)]
        assert layer_base[l + 1] - layer_base[l] == B * sum(R) * D
        for h in range(H):
            prev_end = 0
            for s in range(g.S):
                assert past_len[l, h, s] == sum(g.n[t] for t in range(s) if keep[l, h, t])
                if keep[l, h, s]:
                    assert seg_off[l, h, s] == prev_end
                    prev_end += g.n[s]
                else:
                    assert seg_off[l, h, s] == -1


def test_compaction_identity_coded():
    """Source words encode their (l, b, h, t, d); every destination word must
    decode to a token of a kept scale, each exactly once, in (h, s, raster) order."""
    sides = SIDES_TINY
    g = _geom(sides)
    L, B, H, D = 2, 2, 3, 8
    T = g.T
    ids = np.arange(L * B * H * T, dtype=np.int64).reshape(L, B, H, T)
    kd = np.zeros((L, B, H, T, D), dtype=np.uint16)
    vd = np.zeros((L, B, H, T, D), dtype=np.uint16)
    for d in range(D):
        kd[..., d] = (ids * 8 + d) & 0xFFFF          # 1860 rows * 8 < 65536
        vd[..., d] = (0xFFFF - (ids * 8 + d)) & 0xFFFF
    keep = np.random.default_rng(11).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    head_off, seg_off, past_len, layer_base = oracle.build_offsets(keep, sides, B, D)
    kc, vc = oracle.compact_kv(kd, vd, keep, sides, head_off, seg_off, layer_base)
    assert np.array_equal(vc, (0xFFFF - kc.astype(np.int64)).astype(np.uint16))
    rows = kc.reshape(-1, D)
    assert np.all(rows[:, 1:] - rows[:, :1] == np.arange(1, D, dtype=np.uint16)[None, :])
    decoded = rows[:, 0].astype(np.int64) // 8
    pos = 0
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for s in range(g.S):
                    if keep[l, h, s]:
                        for t in range(g.off[s], g.off[s] + g.n[s]):
                            lb, bb, hh, tt = np.unravel_index(decoded[pos], (L, B, H, T))
                            assert (lb, bb, hh, tt) == (l, b, h, t)
                            pos += 1
    assert pos == rows.shape[0]


# ---------------------------------------------------------------- planted mistakes

def _mutant_checks(monkeypatch, patch):
    """Apply a planted mistake to the oracle and report which pins fail."""
    patch(monkeypatch)
    failures = 0
    for fn in (test_mass_rows_sum_to_one_and_scas_column_sums, test_bias_only_closed_form,
               test_block_causal_matches_library_attention_with_mask,
               test_pruned_matches_library_attention_with_keep_mask,
               test_scale_indicator_values_reproduce_mass):
        try:
            fn()
        except AssertionError:
            failures += 1
    return failures


def _patch_no_tau(mp):
    orig = oatt.attend
    mp.setattr(oatt, "attend", lambda q, k, v, tau, cb, D: orig(q, k, v, 1.0, cb, D))


def _patch_bias_sign(mp):
    orig = oatt.attend
    mp.setattr(oatt, "attend", lambda q, k, v, tau, cb, D: orig(q, k, v, tau, -cb, D))


def _patch_mask_off_by_one(mp):
    G = oatt.ScaleGeometry

    class Shifted(G):
        def __init__(self, sides):
            super().__init__(sides)
            self.L = [self.L[min(k + 1, self.S - 1)] for k in range(self.S)]
    mp.setattr(oatt, "ScaleGeometry", Shifted)


def _patch_transposed_scale(mp):
    orig = oatt._col_bias
    mp.setattr(oatt, "_col_bias", lambda g, b, ks: orig(g, b, list(reversed(list(ks)))))


@pytest.mark.parametrize("patch", [_patch_no_tau, _patch_bias_sign, _patch_mask_off_by_one,
                                   _patch_transposed_scale])
def test_planted_mistakes_are_caught(monkeypatch, patch):
    assert _mutant_checks(monkeypatch, patch) >= 1


# ---------------------------------------------------------------- generation order

def test_appending_every_scale_reproduces_compaction():
    sides = SIDES_TINY
    g = _geom(sides)
    L, B, H, D = 2, 2, 3, 8
    kd = normal_bf16_bits(derive_key(77, 1), (L, B, H, g.T, D))
    vd = normal_bf16_bits(derive_key(77, 2), (L, B, H, g.T, D))
    keep = np.random.default_rng(77).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kref, vref = oracle.compact_kv(kd, vd, keep, sides, ho, so, lb)
    kc = np.zeros(int(lb[-1]), dtype=np.uint16)
    vc = np.zeros(int(lb[-1]), dtype=np.uint16)
    for k in range(g.S):
        sl = slice(g.off[k], g.off[k] + g.n[k])
        oracle.append_scale(kc, vc, np.ascontiguousarray(kd[:, :, :, sl]), np.ascontiguousarray(vd[:, :, :, sl]),
                            keep, sides, ho, so, lb, k)
    assert np.array_equal(kc, kref) and np.array_equal(vc, vref)


def test_cache_size_accounting_closed_forms():
    sides = SIDES_TINY
    g = _geom(sides)
    L, H, B, D = 3, 4, 2, 64
    full = np.ones((L, H, g.S), dtype=np.uint8)
    sz = oracle.cache_size_after_layer(full, sides, B, D)
    per = H * B * D * 4
    for k in range(g.S):
        for l in range(L):
            assert sz[k, l] == L * g.off[k] * per + (l + 1) * g.n[k] * per
    keep = np.random.default_rng(3).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    sz = oracle.cache_size_after_layer(keep, sides, B, D)
    assert np.all(np.diff(sz.ravel()) >= 0)
    _, _, _, lb = oracle.build_offsets(keep, sides, B, D)
    assert sz[-1, -1] == 4 * int(lb[-1])


# ---------------------------------------------------------------- ranking stability

def test_rank_stability_pins():
    from scipy.stats import spearmanr
    sides = SIDES_TINY
    rng = np.random.default_rng(21)
    a = rng.uniform(size=(2, 3, 7))
    b = a + 0.1 * rng.standard_normal(size=a.shape)
    b[0, 0, 2:4] = b[0, 0, 5]                     # ties
    sp, jc = oracle.rank_stability(a, b, sides, 5000, 2)
    ref = spearmanr(a[:, :, 2:].ravel(), b[:, :, 2:].ravel()).correlation
    assert abs(sp - ref) < 1e-12
    sp1, jc1 = oracle.rank_stability(a, a, sides, 5000, 2)
    assert abs(sp1 - 1.0) < 1e-12 and jc1 == 1.0
    sp2, _ = oracle.rank_stability(a, -a, sides, 5000, 2)
    assert abs(sp2 + 1.0) < 1e-12
    assert 0.0 <= jc <= 1.0


# ---------------------------------------------------------------- time-varying schedule

@pytest.mark.parametrize("budget", [10000, 5000, 2500, 1200])
def test_early_pruning_schedule_brute_force(budget):
    """N_k is the smallest non-decreasing prefix length keeping every step's
    retained cache within the absolute budget; evictions follow the O_i."""
    sides = SIDES_TINY
    g = _geom(sides)
    L, H, n_sinks = 2, 3, 2
    LH = L * H
    scas = np.round(np.random.default_rng(budget).uniform(size=(L, H, g.S)), 2)
    prefix, evict = oracle.early_pruning_schedule(scas, sides, budget, n_sinks)
    F = LH * g.T
    prev = 0
    for k in range(g.S):
        def retained(N):
            return sum(LH * g.n[i] for i in range(min(n_sinks, k + 1))) + \
                sum((LH - N) * g.n[i] for i in range(n_sinks, k + 1))
        feasible = [N for N in range(prev, LH + 1) if retained(N) * 10000 <= budget * F]
        want = feasible[0] if feasible else LH
        if k < n_sinks:
            want = 0
        assert prefix[k] == want, (k, prefix[k], want)
        prev = max(prev, prefix[k])
        keep_k = oracle.keep_after_step(evict, k)
        held = int((keep_k * np.array(g.n)[None, None, :]).sum())
        if feasible:
            assert held * 10000 <= budget * F
        # evicted pairs of scale i are exactly the N_k least dependent (l, h) on i
        for i in range(n_sinks, k + 1):
            gone = {lh for lh in range(LH) if not keep_k.reshape(LH, g.S)[lh, i]}
            order = sorted(range(LH), key=lambda lh: (scas.reshape(LH, g.S)[lh, i], lh))
            assert gone == set(order[:prefix[k]])
    if budget == 10000:
        assert np.all(evict == 255)


# ---------------------------------------------------------------- int8 retained cache

def test_int8_block_quantisation_pins():
    from synth import f32_to_bf16_bits
    rng = np.random.default_rng(4)
    x = f32_to_bf16_bits(rng.standard_normal((300, 16)).astype(np.float32) * 3)
    codes, a = oracle.quantize_block(x)
    back = bf16_bits_to_f32(oracle.dequantize_block(codes, a)).astype(np.float64)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    bound = a.astype(np.float64)[None, :] / 254.0 + np.abs(back) * 2.0 ** -8
    assert np.all(np.abs(back - xf) <= bound + 1e-12)
    assert np.all(np.abs(codes.astype(np.int64)).max(axis=0) == 127)   # the absmax element maps to +-127
    # integers in [-127, 127] with absmax 127: scale 1, exact round trip
    ints = rng.integers(-127, 128, size=(50, 8)).astype(np.float32)
    ints[0] = 127.0
    xi = f32_to_bf16_bits(ints)
    ci, ai = oracle.quantize_block(xi)
    assert np.array_equal(ci.astype(np.float32), ints) and np.array_equal(oracle.dequantize_block(ci, ai), xi)
    # zero block
    cz, az = oracle.quantize_block(np.zeros((4, 8), dtype=np.uint16))
    assert not cz.any() and not az.any() and not oracle.dequantize_block(cz, az).any()


# ---------------------------------------------------------------- further pins

def test_scas_from_mass_divides_by_the_call_count():
    """Several calibration calls accumulate into one mass table; dividing by
    the call count gives the mean of the per-call S-CAS; k copies of one table
    leave S-CAS unchanged; a hand-built table gives its closed form."""
    sides = SIDES_TINY
    g = _geom(sides)
    Ms = []
    for tag in (31, 32, 33):
        q, k, v = _qkv(2, 2, g.T, 16, tag=tag)
        _, mass = oracle.block_causal_attention(q, k, v, sides, np.array([0.7, 1.6]), None)
        Ms.append(oracle.scas_mass(mass, sides))
    got = oracle.scas_from_mass(Ms[0] + Ms[1] + Ms[2], 3)
    want = (oracle.scas_from_mass(Ms[0]) + oracle.scas_from_mass(Ms[1]) + oracle.scas_from_mass(Ms[2])) / 3.0
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=0)
    np.testing.assert_allclose(oracle.scas_from_mass(4.0 * Ms[0], 4), oracle.scas_from_mass(Ms[0]), rtol=1e-15,
                               atol=0)
    # M[h][s][k] = (h + 1) * (s + 1) * (k + 1) for s <= k: with 2 calls,
    # S-CAS[h][s] = (h + 1) (s + 1) / 2 * sum_{k = s+1}^{S-1} (k + 1)
    S = g.S
    M = np.zeros((2, S, S))
    for h in range(2):
        for s in range(S):
            for kk in range(s, S):
                M[h, s, kk] = (h + 1) * (s + 1) * (kk + 1)
    sc = oracle.scas_from_mass(M, 2)
    for h in range(2):
        for s in range(S):
            tail = (S * (S + 1)) // 2 - ((s + 1) * (s + 2)) // 2      # sum of k + 1 over k = s+1 .. S-1
            assert sc[h, s] == (h + 1) * (s + 1) * tail / 2.0


def test_rank_stability_closed_forms():
    """Candidates of equal size, so a budget fixes how many pairs each run
    drops (4 of 10 here); drop sets and rank vectors are built by hand, so the
    Jaccard overlap and Spearman's rho have closed forms."""
    sides = (1, 2, 2, 2)                # scales 2, 3 are the candidates, 4 tokens each
    L, H, n_sinks = 1, 5, 2
    F = L * H * 13
    budget = 7540                       # 4 drops: 65 - 16 = 49 <= 0.754 * 65 < 53
    assert (F - 16) * 10000 <= budget * F < (F - 12) * 10000
    cand = [(0, h, s) for h in range(H) for s in (2, 3)]

    def scas_from_ranks(ranks):
        sc = np.zeros((L, H, 4))
        for c, r in zip(cand, ranks):
            sc[c] = 0.1 * r + 0.05
        return sc

    a = scas_from_ranks(range(10))                               # drops c0..c3
    # b drops c0, c1, c4, c5: |A & B| = 2, |A | B| = 6; rank shifts d = (0,0,-2,-2,2,2,0,0,0,0)
    b = scas_from_ranks([0, 1, 4, 5, 2, 3, 6, 7, 8, 9])
    sp, jc = oracle.rank_stability(a, b, sides, budget, n_sinks)
    assert jc == 2 / 6
    assert abs(sp - (1.0 - 6.0 * 16 / (10 * 99))) < 1e-12
    # disjoint drop sets: Jaccard 0
    c = scas_from_ranks([4, 5, 6, 7, 0, 1, 2, 3, 8, 9])
    _, jc0 = oracle.rank_stability(a, c, sides, budget, n_sinks)
    assert jc0 == 0.0
    # one run drops a superset of the other's (budget differs only through sizes: use
    # unequal scales) -- with sides (1, 2, 2, 4): scale 3 holds 16 tokens
    sides2 = (1, 2, 2, 4)
    F2 = H * 25
    cand2 = [(0, h, s) for h in range(H) for s in (2, 3)]
    sa = np.zeros((1, H, 4))
    sb = np.zeros((1, H, 4))
    for i, c_ in enumerate(cand2):
        sa[c_] = 1.0 + i                       # lowest: (h0, s2) 4 tok, (h0, s3) 16 tok, (h1, s2) 4 tok, ...
        sb[c_] = 1.0 + (i if c_[2] == 2 else 100 + i)   # all scale-2 pairs rank below every scale-3 pair
    budget2 = ((F2 - 20) * 10000) // F2        # met once 20 tokens are dropped
    da = oracle.build_schedule(sa, sides2, budget2, n_sinks) == 0
    db = oracle.build_schedule(sb, sides2, budget2, n_sinks) == 0
    # a drops (h0,s2), (h0,s3); b drops the scale-2 pairs of h0..h4 (20 tokens)
    assert int(da.sum()) == 2 and int(db.sum()) == 5
    _, jc2 = oracle.rank_stability(sa, sb, sides2, budget2, n_sinks)
    assert jc2 == 1 / 6


def test_quantize_kv_identity_coded():
    """Each block's values are integers times a power of two that encodes the
    block, with one element per channel at +-127 of that unit: codes are then
    the integers exactly and the absmax is 127 units.  Every code must land at
    the compacted position of its (l, b, h, s, t) -- computed here from the
    layout definition itself -- and every absmax entry at [l][b][h][s][d]."""
    from synth import f32_to_bf16_bits
    sides = SIDES_TINY
    g = _geom(sides)
    L, B, H, D = 2, 2, 3, 8
    T = g.T
    keep = np.random.default_rng(12).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    keep[0, 0, :] = 1

    def code(l, b, h, t, d):
        return int((l * 7 + b * 13 + h * 29 + t * 3 + d * 5) % 255) - 127

    def unit(l, b, h, s):
        return 2.0 ** (((l + 2 * b + 3 * h + 5 * s) % 7) - 3)

    dense = [np.zeros((L, B, H, T, D), dtype=np.float32) for _ in range(2)]
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for s in range(g.S):
                    u = unit(l, b, h, s)
                    for t in range(g.off[s], g.off[s] + g.n[s]):
                        for d in range(D):
                            c = code(l, b, h, t, d)
                            if (t - g.off[s]) == d % g.n[s]:
                                c = 127 if (d % 2 == 0) else -127     # the channel's absmax element
                            dense[0][l, b, h, t, d] = c * u
                            dense[1][l, b, h, t, d] = -c * u
    kb, vb = f32_to_bf16_bits(dense[0]), f32_to_bf16_bits(dense[1])
    head_off, seg_off, _, layer_base = oracle.build_offsets(keep, sides, B, D)
    kq, vq, ka, va = oracle.quantize_kv(kb, vb, keep, sides, head_off, seg_off, layer_base)
    R = (keep * np.array(g.n)[None, None, :]).sum(axis=2)          # [L][H] rows per head
    assert kq.size == 2 * 0 + sum(B * int(R[l].sum()) * D for l in range(L))
    base = 0
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for s in range(g.S):
                    if not keep[l, h, s]:
                        assert not ka[l, b, h, s].any() and not va[l, b, h, s].any()
                        continue
                    np.testing.assert_array_equal(ka[l, b, h, s], 127 * unit(l, b, h, s))
                    np.testing.assert_array_equal(va[l, b, h, s], 127 * unit(l, b, h, s))
                    row0 = b * int(R[l].sum()) + int(R[l, :h].sum()) + sum(g.n[t] for t in range(s) if keep[l, h, t])
                    for t in range(g.n[s]):
                        got = kq[base + (row0 + t) * D: base + (row0 + t + 1) * D].astype(np.int64)
                        gotv = vq[base + (row0 + t) * D: base + (row0 + t + 1) * D].astype(np.int64)
                        want = np.array([code(l, b, h, g.off[s] + t, d) if t != d % g.n[s]
                                         else (127 if d % 2 == 0 else -127) for d in range(D)])
                        assert np.array_equal(got, want) and np.array_equal(gotv, -want), (l, b, h, s, t)
        base += B * int(R[l].sum()) * D


@pytest.mark.parametrize("budget", [10000, 6000, 4000, 2500, 1200])
def test_early_pruning_against_explicit_cache(budget):
    """N_k against the definition built out explicitly: for each candidate N
    the retained set after step k is materialised pair by pair (sinks of every
    head; non-sink scales i <= k of the (layer, head) squares outside the
    length-N prefix of O_i, O_i sorted here by (S-CAS, l, h)) and its tokens
    counted; N_k is the smallest N >= N_{k-1} whose set fits the budget, and
    keep_after_step(evict, k) must be exactly that set."""
    sides = (1, 2, 3, 3, 4, 5)
    g = _geom(sides)
    L, H, n_sinks = 2, 3, 2
    LH = L * H
    scas = np.random.default_rng(budget + 1).uniform(size=(L, H, g.S))
    prefix, evict = oracle.early_pruning_schedule(scas, sides, budget, n_sinks)
    F = LH * g.T
    orders = {i: sorted(((l, h) for l in range(L) for h in range(H)), key=lambda lh: (scas[lh[0], lh[1], i], lh))
              for i in range(n_sinks, g.S)}

    def held_set(k, N):
        keep = np.zeros((L, H, g.S), dtype=np.uint8)
        for l in range(L):
            for h in range(H):
                for i in range(k + 1):
                    keep[l, h, i] = 1 if i < n_sinks else int((l, h) not in orders[i][:N])
        return keep

    prev = 0
    for k in range(g.S):
        if k < n_sinks:
            assert prefix[k] == 0
            want = held_set(k, 0)
        else:
            fits = [N for N in range(prev, LH + 1)
                    if int((held_set(k, N) * np.array(g.n)[None, None, :]).sum()) * 10000 <= budget * F]
            assert fits, k
            assert prefix[k] == fits[0], (k, prefix[k], fits[0])
            prev = fits[0]
            want = held_set(k, fits[0])
        assert np.array_equal(oracle.keep_after_step(evict, k), want), k


def test_large_logits_match_library_attention():
    """Logits far outside the range of N(0,1) inputs (rows of q and k scaled to
    give |x| up to a few hundred): the oracle's max-subtracted softmax still
    equals torch's fp64 attention, and masses still sum to one."""
    sides = SIDES_TINY
    g = _geom(sides)
    q, k, v = _qkv(1, 2, g.T, 64, tag=41)
    q[0, :, ::7] *= 24.0
    k[0, :, ::5] *= 16.0
    q[0, 1, 3] = -q[0, 1, 3] * 40.0
    tau = np.array([2.0, 1.5])
    bias = gen_bias(41, 2, g.S).astype(np.float64)
    O, mass = oracle.block_causal_attention(q, k, v, sides, tau, bias)
    sc = np.array(g.scale_of)
    allowed = sc[None, :] <= sc[:, None]
    for h in range(2):
        x = tau[h] * (q[0, h] @ k[0, h].T) / 8.0
        assert np.abs(x).max() > 200.0
        ref = _sdpa_reference(q[0, h], k[0, h], v[0, h], allowed, tau[h], bias[h][sc])
        np.testing.assert_allclose(O[0, h], ref, atol=1e-11, rtol=0)
    np.testing.assert_allclose(mass.sum(axis=3), 1.0, atol=1e-12, rtol=0)


# ---------------------------------------------------------------- 4-bit retained cache

def test_int4_block_quantisation_pins():
    from synth import f32_to_bf16_bits
    rng = np.random.default_rng(44)
    x = f32_to_bf16_bits(rng.standard_normal((300, 16)).astype(np.float32) * 3)
    codes, s_bits = oracle.quantize_block_int4(x)
    s = bf16_bits_to_f32(s_bits).astype(np.float64)
    a = np.abs(bf16_bits_to_f32(x)).max(axis=0).astype(np.float64)
    # s is a / 7 rounded to bf16: within half a bf16 step of it
    assert np.all(np.abs(s - a / 7.0) <= (a / 7.0) * 2.0 ** -8)
    back = bf16_bits_to_f32(oracle.dequantize_block_int4(codes, s_bits)).astype(np.float64)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    assert np.all(np.abs(back - xf) <= s[None, :] / 2.0 + np.abs(back) * 2.0 ** -9 + 1e-12)
    assert np.all(np.abs(codes.astype(np.int64)).max(axis=0) == 7)       # the absmax element maps to +-7
    assert codes.min() >= -7 and codes.max() <= 7
    # the exact product, rounded once: code * s has at most 11 significant bits
    prod = codes.astype(np.float64) * s[None, :]
    assert np.array_equal(oracle.dequantize_block_int4(codes, s_bits),
                          f32_to_bf16_bits(prod.astype(np.float32)))
    # integers in [-7, 7] with absmax 7 on every channel: scale 1, exact round trip
    ints = rng.integers(-7, 8, size=(40, 8)).astype(np.float32)
    ints[0] = 7.0
    xi = f32_to_bf16_bits(ints)
    ci, si = oracle.quantize_block_int4(xi)
    assert np.all(bf16_bits_to_f32(si) == 1.0)
    assert np.array_equal(ci.astype(np.float32), ints) and np.array_equal(oracle.dequantize_block_int4(ci, si), xi)
    # zero block
    cz, sz = oracle.quantize_block_int4(np.zeros((4, 8), dtype=np.uint16))
    assert not cz.any() and not sz.any() and not oracle.dequantize_block_int4(cz, sz).any()


def test_int4_packing_layout():
    """One hand-packed word: codes c0..c7 = -7, -6, 0, 1, 2, 3, 7, -1 give
    nibbles 1, 2, 8, 9, 10, 11, 15, 7; the even channels fill nibbles 0-3 and
    the odd ones nibbles 4-7 -> 0x7B92FA81, stored little-endian."""
    codes = np.array([[-7, -6, 0, 1, 2, 3, 7, -1]], dtype=np.int8)
    packed = oracle.pack_int4(codes)
    assert packed.tolist() == [[0x81, 0xFA, 0x92, 0x7B]]
    rng = np.random.default_rng(45)
    many = rng.integers(-7, 8, size=(33, 64)).astype(np.int8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(many), 64), many)


def test_quantize_kv_int4_identity_coded():
    """As the int8 identity pin: integer codes times a power-of-two unit per
    block, one +-7 element per channel, so the codes are the integers and the
    scale is the unit; every nibble must land at its compacted position."""
    from synth import f32_to_bf16_bits
    sides = SIDES_TINY
    g = _geom(sides)
    L, B, H, D = 2, 2, 3, 8
    T = g.T
    keep = np.random.default_rng(13).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    keep[1, 2, :] = 1

    def code(l, b, h, t, d):
        return int((l * 5 + b * 11 + h * 3 + t * 7 + d * 13) % 15) - 7

    def unit(l, b, h, s):
        return 2.0 ** (((3 * l + b + 2 * h + s) % 9) - 4)

    dense = np.zeros((L, B, H, T, D), dtype=np.float32)
    want_codes = np.zeros((L, B, H, T, D), dtype=np.int64)
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for s in range(g.S):
                    for t in range(g.off[s], g.off[s] + g.n[s]):
                        for d in range(D):
                            c = code(l, b, h, t, d)
                            if (t - g.off[s]) == d % g.n[s]:
                                c = 7 if (d + t) % 2 == 0 else -7
                            want_codes[l, b, h, t, d] = c
                            dense[l, b, h, t, d] = c * unit(l, b, h, s)
    kb = f32_to_bf16_bits(dense)
    vb = f32_to_bf16_bits(-dense)
    head_off, seg_off, _, layer_base = oracle.build_offsets(keep, sides, B, D)
    kq, vq, ks, vs = oracle.quantize_kv_int4(kb, vb, keep, sides, head_off, seg_off, layer_base)
    R = (keep * np.array(g.n)[None, None, :]).sum(axis=2)
    assert 2 * kq.size == sum(B * int(R[l].sum()) * D for l in range(L))
    base = 0
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for s in range(g.S):
                    if not keep[l, h, s]:
                        assert not ks[l, b, h, s].any() and not vs[l, b, h, s].any()
                        continue
                    assert np.all(bf16_bits_to_f32(ks[l, b, h, s]) == unit(l, b, h, s))
                    row0 = b * int(R[l].sum()) + int(R[l, :h].sum()) + sum(g.n[t] for t in range(s) if keep[l, h, t])
                    for t in range(g.n[s]):
                        lo = (base + (row0 + t) * D) // 2
                        got_k = oracle.unpack_int4(kq[lo:lo + D // 2], D)[0]
                        got_v = oracle.unpack_int4(vq[lo:lo + D // 2], D)[0]
                        want = want_codes[l, b, h, g.off[s] + t]
                        assert np.array_equal(got_k, want) and np.array_equal(got_v, -want), (l, b, h, s, t)
        base += B * int(R[l].sum()) * D


# ---------------------------------------------------------------- 3-bit retained cache

def test_int3_block_quantisation_pins():
    from synth import f32_to_bf16_bits
    rng = np.random.default_rng(46)
    x = f32_to_bf16_bits(rng.standard_normal((300, 16)).astype(np.float32) * 3)
    codes, s_bits = oracle.quantize_block_int3(x)
    s = bf16_bits_to_f32(s_bits).astype(np.float64)
    a = np.abs(bf16_bits_to_f32(x)).max(axis=0).astype(np.float64)
    # s is a / 3 rounded to bf16: within half a bf16 step of it
    assert np.all(np.abs(s - a / 3.0) <= (a / 3.0) * 2.0 ** -8)
    back = bf16_bits_to_f32(oracle.dequantize_block_int3(codes, s_bits)).astype(np.float64)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    assert np.all(np.abs(back - xf) <= s[None, :] / 2.0 + np.abs(back) * 2.0 ** -9 + 1e-12)
    assert np.all(np.abs(codes.astype(np.int64)).max(axis=0) == 3)       # the absmax element maps to +-3
    assert codes.min() >= -3 and codes.max() <= 3
    # the exact product, rounded once: code * s has at most 10 significant bits
    prod = codes.astype(np.float64) * s[None, :]
    assert np.array_equal(oracle.dequantize_block_int3(codes, s_bits),
                          f32_to_bf16_bits(prod.astype(np.float32)))
    # integers in [-3, 3] with absmax 3 on every channel: scale 1, exact round trip
    ints = rng.integers(-3, 4, size=(40, 8)).astype(np.float32)
    ints[0] = -3.0
    xi = f32_to_bf16_bits(ints)
    ci, si = oracle.quantize_block_int3(xi)
    assert np.all(bf16_bits_to_f32(si) == 1.0)
    assert np.array_equal(ci.astype(np.float32), ints) and np.array_equal(oracle.dequantize_block_int3(ci, si), xi)
    # halves round to even: with scale 1, 0.5 -> 0, 1.5 -> 2, -2.5 -> -2
    xh = f32_to_bf16_bits(np.array([[0.5, 1.5, -2.5, 3.0], [3.0, -3.0, 3.0, -3.0]], dtype=np.float32))
    ch, sh = oracle.quantize_block_int3(xh)
    assert np.all(bf16_bits_to_f32(sh) == 1.0) and ch[0].tolist() == [0, 2, -2, 3]
    # zero block
    cz, sz = oracle.quantize_block_int3(np.zeros((4, 8), dtype=np.uint16))
    assert not cz.any() and not sz.any() and not oracle.dequantize_block_int3(cz, sz).any()


def test_int3_packing_layout():
    """One hand-packed group: codes c0..c7 = -3, -2, -1, 0, 1, 2, 3, 0 give
    fields 1, 2, 3, 4, 5, 6, 7, 4 at bits 3j; written high field first that is
    100 111 110 101 100 011 010 001 = 0x9F58D1, stored little-endian.  A second
    group follows in the next three bytes."""
    codes = np.array([[-3, -2, -1, 0, 1, 2, 3, 0, 3, 3, 3, 3, 3, 3, 3, 3]], dtype=np.int8)
    packed = oracle.pack_int3(codes)
    assert packed.tolist() == [[0xD1, 0x58, 0x9F, 0xFF, 0xFF, 0xFF]]   # eight 7-fields = 24 ones
    rng = np.random.default_rng(47)
    many = rng.integers(-3, 4, size=(33, 64)).astype(np.int8)
    assert np.array_equal(oracle.unpack_int3(oracle.pack_int3(many), 64), many)


def test_quantize_kv_int3_identity_coded():
    """Integer codes in [-3, 3] times a power-of-two unit per block, one +-3
    element per channel: the codes are the integers, the scale the unit, and
    every 3-bit field must land at its compacted position (byte 3 e / 8)."""
    from synth import f32_to_bf16_bits
    sides = SIDES_TINY
    g = _geom(sides)
    L, B, H, D = 2, 2, 3, 16
    T = g.T
    keep = np.random.default_rng(14).integers(0, 2, size=(L, H, g.S)).astype(np.uint8)
    keep[1, 2, :] = 1

    def code(l, b, h, t, d):
        return int((l * 5 + b * 11 + h * 3 + t * 7 + d * 13) % 7) - 3

    def unit(l, b, h, s):
        return 2.0 ** (((3 * l + b + 2 * h + s) % 9) - 4)

    dense = np.zeros((L, B, H, T, D), dtype=np.float32)
    want_codes = np.zeros((L, B, H, T, D), dtype=np.int64)
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for s in range(g.S):
                    for t in range(g.off[s], g.off[s] + g.n[s]):
                        for d in range(D):
                            c = code(l, b, h, t, d)
                            if (t - g.off[s]) == d % g.n[s]:
                                c = 3 if (d + t) % 2 == 0 else -3
                            want_codes[l, b, h, t, d] = c
                            dense[l, b, h, t, d] = c * unit(l, b, h, s)
    kb = f32_to_bf16_bits(dense)
    vb = f32_to_bf16_bits(-dense)
    head_off, seg_off, _, layer_base = oracle.build_offsets(keep, sides, B, D)
    kq, vq, ks, vs = oracle.quantize_kv_int3(kb, vb, keep, sides, head_off, seg_off, layer_base)
    R = (keep * np.array(g.n)[None, None, :]).sum(axis=2)
    assert 8 * kq.size == 3 * sum(B * int(R[l].sum()) * D for l in range(L))
    base = 0
    for l in range(L):
        for b in range(B):
            for h in range(H):
                for s in range(g.S):
                    if not keep[l, h, s]:
                        assert not ks[l, b, h, s].any() and not vs[l, b, h, s].any()
                        continue
                    assert np.all(bf16_bits_to_f32(ks[l, b, h, s]) == unit(l, b, h, s))
                    row0 = b * int(R[l].sum()) + int(R[l, :h].sum()) + sum(g.n[t] for t in range(s) if keep[l, h, t])
                    for t in range(g.n[s]):
                        lo = 3 * (base + (row0 + t) * D) // 8
                        got_k = oracle.unpack_int3(kq[lo:lo + 3 * D // 8], D)[0]
                        got_v = oracle.unpack_int3(vq[lo:lo + 3 * D // 8], D)[0]
                        want = want_codes[l, b, h, g.off[s] + t]
                        assert np.array_equal(got_k, want) and np.array_equal(got_v, -want), (l, b, h, s, t)
        base += B * int(R[l].sum()) * D
