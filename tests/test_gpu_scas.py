"""GPU vs oracle: S-CAS calibration attention (attention output and the
per-(head, source scale, query scale) mass), S-CAS and the schedule built on it."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from synth import SIDES_TINY, SIDES_1024
from tests.helpers import bits_of, check_status, dev_bf16, f64, status_word

pytestmark = pytest.mark.gpu

O_ATOL = 2e-2
MASS_RTOL = 1e-3   # relative only: entries s > k are exactly 0 on both sides


def _calib_inputs(sides, B, H, D, seed, with_bias):
    T = synth.n_tokens(sides)
    bits = [synth.normal_bf16_bits(synth.derive_key(60, seed, i), (B, H, T, D)) for i in range(3)]
    tau = synth.gen_tau(seed, H)
    bias = synth.gen_bias(seed, H, len(sides)) if with_bias else None
    return bits, tau, bias


def _gpu_calib(bits, sides, tau, bias, want_out=True):
    q, k, v = (dev_bf16(b) for b in bits)
    B, H, T, D = q.shape
    S = len(sides)
    mass = torch.zeros((H, S, S), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q) if want_out else None
    st = status_word()
    vark.vark_scas_accumulate(q, k, v, sides, torch.from_numpy(tau).cuda(),
                              None if bias is None else torch.from_numpy(bias).cuda(), mass, out, st)
    check_status(st)
    return mass.cpu().numpy().astype(np.float64), (None if out is None else f64(bits_of(out)))


@pytest.mark.parametrize("with_bias", [False, True])
def test_scas_tiny_full_parity(with_bias):
    sides = SIDES_TINY
    bits, tau, bias = _calib_inputs(sides, 4, 4, 64, 1, with_bias)
    M_gpu, O_gpu = _gpu_calib(bits, sides, tau, bias)
    q, k, v = (f64(b) for b in bits)
    O_ref, mass = oracle.block_causal_attention(q, k, v, sides, tau.astype(np.float64),
                                                None if bias is None else bias.astype(np.float64))
    M_ref = oracle.scas_mass(mass, sides)
    assert np.abs(O_gpu - O_ref).max() <= O_ATOL
    np.testing.assert_allclose(M_gpu, M_ref, rtol=MASS_RTOL)
    # S-CAS through the library's host finaliser vs the oracle's
    sc_gpu = vark.vark_scas_finalize(M_gpu.astype(np.float32)[None])
    sc_ref = oracle.scas_from_mass(M_ref[None])
    np.testing.assert_allclose(sc_gpu, sc_ref, rtol=MASS_RTOL)


def _gaps_clear_along_drop_order(sc_ref, sc_gpu, keep_ref, n_sinks, gap=1e-4):
    """The schedule-parity condition where it decides the result.  The greedy
    walk drops candidates in ascending (S-CAS, l, h, s) order and stops at the
    first prefix that meets the budget, so the order of every candidate up to
    and including the first retained one matters (a near-tie anywhere in that
    prefix can change where the walk stops).  Along that prefix two neighbours
    must be more than `gap` apart, or an exact tie on BOTH sides (e.g. the last
    scale, which no later scale reads, scores exactly 0): exact ties are broken
    by index identically by both builders."""
    L, H, S = sc_ref.shape
    cand = sorted((float(sc_ref[l, h, s]), l, h, s) for l in range(L) for h in range(H) for s in range(n_sinks, S))
    n_drop = int((keep_ref[:, :, n_sinks:] == 0).sum())
    prefix = cand[:n_drop + 1]
    for (a, *ia), (b, *ib) in zip(prefix, prefix[1:]):
        if a == b:
            if sc_gpu[tuple(ia)] != sc_gpu[tuple(ib)]:
                return False
        elif b - a <= gap:
            return False
    return True


def _schedule_parity(M_gpu, M_ref, sides, budgets, n_sinks=2):
    sc_gpu = vark.vark_scas_finalize(np.stack(M_gpu).astype(np.float32))
    sc_ref = oracle.scas_from_mass(np.stack(M_ref))
    np.testing.assert_allclose(sc_gpu, sc_ref, rtol=MASS_RTOL)
    checked = 0
    for budget in budgets:
        keep_ref = oracle.build_schedule(sc_ref, sides, budget, n_sinks)
        keep_gpu = vark.vark_build_schedule(sc_gpu, sides, budget, n_sinks)
        # the builder itself is exact on the same input
        assert np.array_equal(vark.vark_build_schedule(sc_ref, sides, budget, n_sinks), keep_ref)
        # the seeds are chosen so that the condition holds: the comparison runs
        assert _gaps_clear_along_drop_order(sc_ref, sc_gpu, keep_ref, n_sinks), budget
        assert int((keep_ref[:, :, n_sinks:] == 0).sum()) > 0
        assert np.array_equal(keep_gpu, keep_ref), budget
        checked += 1
    assert checked == len(budgets)


def test_scas_tiny_schedule_parity():
    """GPU S-CAS -> host schedule equals the oracle's schedule bit for bit
    (3 layers x 4 heads, tiny scales, budgets from 55% down to 20%: every
    budget drops pairs beyond the last scale's structural zeros)."""
    sides = SIDES_TINY
    L, H, B = 3, 4, 4
    M_gpu, M_ref = [], []
    for l in range(L):
        bits, tau, _ = _calib_inputs(sides, B, H, 64, 37 + l, False)
        Mg, _ = _gpu_calib(bits, sides, tau, None, want_out=False)
        q, k, v = (f64(b) for b in bits)
        _, mass = oracle.block_causal_attention(q, k, v, sides, tau.astype(np.float64), None)
        M_gpu.append(Mg)
        M_ref.append(oracle.scas_mass(mass, sides))
    _schedule_parity(M_gpu, M_ref, sides, (5500, 5000, 4000, 3000, 2000))


@pytest.mark.slow
def test_scas_1024_schedule_parity():
    """1024^2 scales with bias, 2 layers x 4 heads x 2 calibration seeds: GPU
    calibration (with O, as in the benchmark step) -> S-CAS -> schedule at 10%
    and 4% equals the oracle's; the mass matches in full."""
    sides = SIDES_1024
    L, H, B = 2, 4, 2
    M_gpu, M_ref = [], []
    for l in range(L):
        bits, tau, bias = _calib_inputs(sides, B, H, 128, 8 + l, True)
        Mg, _ = _gpu_calib(bits, sides, tau, bias, want_out=True)
        q, k, v = (f64(b) for b in bits)
        _, mass = oracle.block_causal_attention(q, k, v, sides, tau.astype(np.float64), bias.astype(np.float64))
        Mr = oracle.scas_mass(mass, sides)
        np.testing.assert_allclose(Mg, Mr, rtol=MASS_RTOL)
        M_gpu.append(Mg)
        M_ref.append(Mr)
    _schedule_parity(M_gpu, M_ref, sides, (1000, 400))


def test_scas_1024_two_seeds_two_heads_full_parity():
    sides = SIDES_1024
    bits, tau, bias = _calib_inputs(sides, 2, 2, 128, 2, True)
    M_gpu, O_gpu = _gpu_calib(bits, sides, tau, bias)
    q, k, v = (f64(b) for b in bits)
    O_ref, mass = oracle.block_causal_attention(q, k, v, sides, tau.astype(np.float64), bias.astype(np.float64))
    M_ref = oracle.scas_mass(mass, sides)
    assert np.abs(O_gpu - O_ref).max() <= O_ATOL
    np.testing.assert_allclose(M_gpu, M_ref, rtol=MASS_RTOL)


@pytest.mark.parametrize("sides,B,H,D", [(SIDES_TINY, 4, 4, 64), (SIDES_1024, 2, 2, 128), (SIDES_1024, 3, 1, 64)])
def test_scas_without_output_matches_oracle(sides, B, H, D):
    """S-CAS only (no output buffer): the kernel skips V and PV, and the mass
    still matches the oracle and the with-output run."""
    bits, tau, bias = _calib_inputs(sides, B, H, D, 7 + D, True)
    M_noo, O_none = _gpu_calib(bits, sides, tau, bias, want_out=False)
    assert O_none is None
    M_o, _ = _gpu_calib(bits, sides, tau, bias, want_out=True)
    q, k, v = (f64(b) for b in bits)
    _, mass = oracle.block_causal_attention(q, k, v, sides, tau.astype(np.float64), bias.astype(np.float64))
    M_ref = oracle.scas_mass(mass, sides)
    np.testing.assert_allclose(M_noo, M_ref, rtol=MASS_RTOL)
    np.testing.assert_allclose(M_noo, M_o, rtol=MASS_RTOL)
    S = len(sides)
    for kk in range(S):
        np.testing.assert_allclose(M_noo[:, :kk + 1, kk].sum(axis=1), 1.0, atol=1e-4)


@pytest.mark.slow
def test_scas_calibration_full_size_sampled():
    """16 seeds x 16 heads at 1024^2, inputs made on the device: mass sums to
    one per (h, k); M of one head for every query scale and of another for the
    scales <= 8, and sampled output rows of several scales, against the
    oracle."""
    w = synth.WORKLOADS["calib_1024"]
    sides, H, D, B = w.sides, w.heads, w.head_dim, w.n_seeds
    T = synth.n_tokens(sides)
    S = len(sides)
    g = oracle.ScaleGeometry(sides)
    keys = [synth.qkv_key(w, 0, x, "calib") for x in ("q", "k", "v")]
    q, k, v = (synth.normal_bf16_torch(key, (B, H, T, D), device="cuda") for key in keys)
    tau = synth.gen_tau(synth.layer_seed(w, 0), H)
    bias = synth.gen_bias(synth.layer_seed(w, 0), H, S)
    mass = torch.zeros((H, S, S), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    st = status_word()
    vark.vark_scas_accumulate(q, k, v, sides, torch.from_numpy(tau).cuda(), torch.from_numpy(bias).cuda(), mass,
                              out, st)
    check_status(st)
    M = mass.cpu().numpy().astype(np.float64)
    for kk in range(S):
        np.testing.assert_allclose(M[:, :kk + 1, kk].sum(axis=1), 1.0, atol=1e-4)
        assert np.all(M[:, kk + 1:, kk] == 0)
    shape = (B, H, T, D)
    # head 11: M for every query scale (scales 9-12 carry ~98% of the work);
    # head 0: the scales <= 8
    for h, n_k in ((11, S), (0, 9)):
        Lk = g.L[n_k - 1]
        acc = np.zeros((S, n_k))
        for b in range(B):
            kb = f64(synth.rows_bf16_bits(keys[1], shape, (b, h), 0, Lk))
            vb = f64(synth.rows_bf16_bits(keys[2], shape, (b, h), 0, Lk))
            qb = f64(synth.rows_bf16_bits(keys[0], shape, (b, h), 0, Lk))
            for kk in range(n_k):
                r0, r1 = g.off[kk], g.L[kk]
                _, m = oracle.attention_rows(qb[r0:r1], kb, vb, sides, kk, float(tau[h]), bias[h].astype(np.float64))
                acc[:, kk] += m.sum(axis=0) / (B * g.n[kk])
        np.testing.assert_allclose(M[h, :, :n_k], acc, rtol=MASS_RTOL)
    rng = np.random.default_rng(0)
    for kk in (0, 5, 9, 12):
        b, h = int(rng.integers(B)), int(rng.integers(H))
        rows = np.unique(np.concatenate([[0, g.n[kk] - 1], rng.integers(0, g.n[kk], size=6)]))
        kb = f64(synth.rows_bf16_bits(keys[1], shape, (b, h), 0, g.L[kk]))
        vb = f64(synth.rows_bf16_bits(keys[2], shape, (b, h), 0, g.L[kk]))
        qb = f64(synth.rows_bf16_bits(keys[0], shape, (b, h), g.off[kk], g.L[kk]))[rows]
        o_ref, _ = oracle.attention_rows(qb, kb, vb, sides, kk, float(tau[h]), bias[h].astype(np.float64))
        o_gpu = out[b, h, g.off[kk] + torch.from_numpy(rows).cuda()].float().cpu().numpy()
        assert np.abs(o_gpu - o_ref).max() <= O_ATOL
