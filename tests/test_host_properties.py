"""Property tests of the library's host-side builders against the oracle on
randomly drawn small problems, edge cases included: no sinks or every scale a
sink, one scale, zero and full budgets, heavy ties (values drawn from a small
set, signed zeros).  Both sides must agree exactly, including on which inputs
are infeasible."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import kv_cache_compression_cas_b200 as vark
import oracle

SETTINGS = dict(max_examples=250, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw):
    S = draw(st.integers(1, 6))
    sides = tuple(draw(st.lists(st.integers(1, 6), min_size=S, max_size=S)))
    L = draw(st.integers(1, 3))
    H = draw(st.integers(1, 4))
    pool = [-0.0, 0.0, 0.25, 0.5, 0.5000000001, 1.0, 3.0]
    vals = draw(st.lists(st.sampled_from(pool), min_size=L * H * S, max_size=L * H * S))
    scas = np.array(vals, dtype=np.float64).reshape(L, H, S)
    budget = draw(st.one_of(st.sampled_from([0, 1, 9999, 10000]), st.integers(0, 10000)))
    n_sinks = draw(st.integers(0, S))
    return sides, scas, budget, n_sinks


def _both(fn_lib, fn_ref):
    try:
        ref = fn_ref()
    except oracle.BudgetError:
        with pytest.raises(vark.VarkError) as e:
            fn_lib()
        assert e.value.status == -4
        return None, None
    return fn_lib(), ref


@settings(**SETTINGS)
@given(problems())
def test_static_schedule_matches_oracle(prob):
    sides, scas, budget, n_sinks = prob
    got, ref = _both(lambda: vark.vark_build_schedule(scas, sides, budget, n_sinks),
                     lambda: oracle.build_schedule(scas, sides, budget, n_sinks))
    if ref is not None:
        assert np.array_equal(got, ref)
        # sinks are never dropped; the kept tokens meet the budget
        assert np.all(got[:, :, :n_sinks] == 1)
        g = oracle.ScaleGeometry(sides)
        kept = int((got * np.array(g.n)[None, None, :]).sum())
        assert kept * 10000 <= budget * got.shape[0] * got.shape[1] * g.T or budget == 10000


@settings(**SETTINGS)
@given(problems())
def test_early_pruning_schedule_matches_oracle(prob):
    sides, scas, budget, n_sinks = prob
    got, ref = _both(lambda: vark.vark_build_early_pruning_schedule(scas, sides, budget, n_sinks),
                     lambda: oracle.early_pruning_schedule(scas, sides, budget, n_sinks))
    if ref is not None:
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


@settings(**SETTINGS)
@given(problems(), st.integers(1, 3), st.sampled_from([8, 64, 128]))
def test_cache_accounting_matches_oracle(prob, B, D):
    sides, scas, budget, n_sinks = prob
    keep = (scas > 0.4).astype(np.uint8)
    assert np.array_equal(vark.vark_cache_size_after_layer(keep, sides, B, D),
                          oracle.cache_size_after_layer(keep, sides, B, D))


@settings(**SETTINGS)
@given(problems(), st.integers(0, 2 ** 31 - 1))
def test_rank_stability_matches_oracle(prob, seed):
    sides, scas, budget, n_sinks = prob
    if n_sinks == len(sides):
        return   # no candidate pairs to rank
    rng = np.random.default_rng(seed)
    other = np.round(scas + rng.choice([0.0, 0.25, -0.25], size=scas.shape), 2)
    got, ref = _both(lambda: vark.vark_rank_stability(scas, other, sides, budget, n_sinks),
                     lambda: oracle.rank_stability(scas, other, sides, budget, n_sinks))
    if ref is not None:
        assert got[1] == ref[1]
        assert (np.isnan(got[0]) and np.isnan(ref[0])) or abs(got[0] - ref[0]) < 1e-12
