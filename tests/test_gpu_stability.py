"""GPU vs oracle: ranking stability of S-CAS across calibration runs ([HeatKV]
Results: rankings stay stable with a small calibration set; [Review] Figure 6
caption: stability of head-scale rankings across calibration runs).

Two calibration runs on disjoint seed halves, 3 layers x 4 heads, tiny scale
list with bias: the GPU calibration of each half feeds the library's S-CAS
finaliser and vark_rank_stability; the oracle computes both halves' S-CAS in
fp64 and its own ranking stability.  With every neighbouring pair of distinct
candidate values more than 1e-4 apart (the seeds are chosen so, and the test
asserts it), the two sides rank the candidates identically, so Spearman's rho
and the drop-set Jaccard overlap must agree exactly."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from synth import SIDES_TINY
from tests.helpers import check_status, dev_bf16, f64, status_word

pytestmark = pytest.mark.gpu

L, H, B, D = 3, 4, 4, 64
N_SINKS = 2


def _half(seed):
    sides = SIDES_TINY
    S, T = len(sides), synth.n_tokens(sides)
    M_gpu, M_ref = [], []
    for l in range(L):
        bits = [synth.normal_bf16_bits(synth.derive_key(61, seed, l, i), (B, H, T, D)) for i in range(3)]
        tau = synth.gen_tau(100 + l, H)           # the model's per-layer parameters, shared by both halves
        bias = synth.gen_bias(100 + l, H, S)
        q, k, v = (dev_bf16(b) for b in bits)
        mass = torch.zeros((H, S, S), dtype=torch.float32, device="cuda")
        st = status_word()
        vark.vark_scas_accumulate(q, k, v, sides, torch.from_numpy(tau).cuda(), torch.from_numpy(bias).cuda(),
                                  mass, None, st)
        check_status(st)
        M_gpu.append(mass.cpu().numpy())
        _, m = oracle.block_causal_attention(*(f64(b) for b in bits), sides, tau.astype(np.float64),
                                             bias.astype(np.float64))
        M_ref.append(oracle.scas_mass(m, sides))
    return vark.vark_scas_finalize(np.stack(M_gpu)), oracle.scas_from_mass(np.stack(M_ref))


def _clear(sc_ref, sc_gpu, gap=1e-4):
    """Distinct candidate values more than `gap` apart, exact ties tied on both sides."""
    ref = sc_ref[:, :, N_SINKS:].ravel()
    gpu = sc_gpu[:, :, N_SINKS:].ravel()
    order = np.argsort(ref, kind="stable")
    for i, j in zip(order, order[1:]):
        if ref[i] == ref[j]:
            if gpu[i] != gpu[j]:
                return False
        elif ref[j] - ref[i] <= gap:
            return False
    return True


@pytest.mark.parametrize("budget_bp", [5000, 4000, 2500])
def test_rank_stability_gpu_calibration_matches_oracle(budget_bp):
    sides = SIDES_TINY
    gpu_a, ref_a = _half(1)
    gpu_b, ref_b = _half(2)
    np.testing.assert_allclose(gpu_a, ref_a, rtol=1e-3)
    np.testing.assert_allclose(gpu_b, ref_b, rtol=1e-3)
    assert _clear(ref_a, gpu_a) and _clear(ref_b, gpu_b)
    sp_gpu, jc_gpu = vark.vark_rank_stability(gpu_a, gpu_b, sides, budget_bp, N_SINKS)
    sp_ref, jc_ref = oracle.rank_stability(ref_a, ref_b, sides, budget_bp, N_SINKS)
    assert abs(sp_gpu - sp_ref) <= 1e-12
    assert jc_gpu == jc_ref
    assert 0.9 < sp_ref < 1.0               # the halves differ, but rank the pairs alike
    # the library's host statistic equals the oracle's on the same input
    sp_same, jc_same = oracle.rank_stability(gpu_a, gpu_b, sides, budget_bp, N_SINKS)
    assert abs(sp_gpu - sp_same) <= 1e-12 and jc_gpu == jc_same
