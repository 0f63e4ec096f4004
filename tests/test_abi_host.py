"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every symbol the header declares, the host-only calls (schedule
builder, S-CAS finalisation) agree bit for bit with the oracle, and argument
errors come back as status codes before any device work."""
import ctypes

import numpy as np
import pytest

import kv_cache_compression_cas_b200 as vark
import oracle
from synth import SIDES_TINY, SIDES_1024


def test_library_exports_every_header_symbol():
    lib = vark.library()
    names = vark.header_symbols()
    assert {"vark_scas_accumulate", "vark_build_schedule", "vark_build_offsets", "vark_compact_kv",
            "vark_pruned_attention", "vark_scas_finalize", "vark_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert vark.vark_version() >= 10000
    for code in range(-7, 1):
        assert vark.vark_status_string(code).startswith("VARK")


@pytest.mark.parametrize("sides,L,H", [(SIDES_TINY, 1, 4), (SIDES_TINY, 3, 5), (SIDES_1024, 32, 16),
                                       (SIDES_1024, 8, 32)])
def test_schedule_builder_bit_exact_with_oracle(sides, L, H):
    rng = np.random.default_rng(L * 100 + H)
    S = len(sides)
    scas = rng.uniform(0, 1, size=(L, H, S))
    scas[:, :, -1] = 0.0
    for budget in (10000, 9999, 5000, 2000, 1000, 400, 200):
        try:
            ref = oracle.build_schedule(scas, sides, budget, 2)
        except oracle.BudgetError:
            with pytest.raises(vark.VarkError) as e:
                vark.vark_build_schedule(scas, sides, budget, 2)
            assert e.value.status == -4
            continue
        got = vark.vark_build_schedule(scas, sides, budget, 2)
        assert np.array_equal(got, ref), budget


def test_schedule_builder_ties_and_sinks():
    sides = SIDES_TINY
    S = len(sides)
    scas = np.round(np.random.default_rng(3).uniform(size=(2, 3, S)), 1)   # many exact ties
    for n_sinks in (0, 1, 2, 3):
        for budget in (9000, 6000, 3000):
            try:
                ref = oracle.build_schedule(scas, sides, budget, n_sinks)
            except oracle.BudgetError:
                continue
            assert np.array_equal(vark.vark_build_schedule(scas, sides, budget, n_sinks), ref)
    z = np.zeros((2, 3, S))
    assert np.array_equal(vark.vark_build_schedule(z, sides, 7000, 2), oracle.build_schedule(z, sides, 7000, 2))


def test_scas_finalize_matches_oracle():
    rng = np.random.default_rng(9)
    M = rng.uniform(0, 1, size=(4, 5, 13, 13)).astype(np.float32)
    for n_calls in (1, 3):
        got = vark.vark_scas_finalize(M, n_calls)
        ref = oracle.scas_from_mass(M.astype(np.float64), n_calls)
        np.testing.assert_allclose(got, ref, rtol=1e-15, atol=0)


def test_argument_errors_are_status_codes():
    lib = vark.library()
    sides = (ctypes.c_int32 * 7)(*SIDES_TINY)
    keep = np.zeros((1, 4, 7), dtype=np.uint8)
    scas = np.zeros((1, 4, 7))
    # host builder
    assert lib.vark_build_schedule(None, 1, 4, 7, sides, 5000, 2, keep.ctypes.data) == -1
    assert lib.vark_build_schedule(scas.ctypes.data, 1, 4, 0, sides, 5000, 2, keep.ctypes.data) == -2
    assert lib.vark_build_schedule(scas.ctypes.data, 1, 4, 7, sides, 10001, 2, keep.ctypes.data) == -1
    assert lib.vark_build_schedule(scas.ctypes.data, 1, 4, 7, sides, 100, 2, keep.ctypes.data) == -4
    bad = scas.copy()
    bad[0, 0, 3] = np.nan
    assert lib.vark_build_schedule(bad.ctypes.data, 1, 4, 7, sides, 5000, 2, keep.ctypes.data) == -1
    assert lib.vark_scas_finalize(None, 1, 4, 7, 1, None) == -1
    # device calls reject bad arguments before touching the device
    p = ctypes.c_void_p(16)
    assert lib.vark_scas_accumulate(None, p, p, 1, 4, 64, 7, sides, p, None, p, None, p, None) == -1
    assert lib.vark_scas_accumulate(p, p, p, 1, 4, 96, 7, sides, p, None, p, None, p, None) == -2
    assert lib.vark_scas_accumulate(p, p, p, 1, 4, 64, 7, sides, p, None, p, None, None, None) == -1
    assert lib.vark_scas_accumulate(ctypes.c_void_p(24), p, p, 1, 4, 64, 7, sides, p, None, p, None, p, None) == -3
    assert lib.vark_pruned_attention(p, p, p, 0, p, p, 1, 4, 7, 64, sides, 9, p, p, p, p, None, p, p, None) == -1
    assert lib.vark_pruned_attention(p, p, p, 0, p, p, 1, 4, 7, 80, sides, -1, p, p, p, p, None, p, p, None) == -2
    assert lib.vark_compact_kv(p, p, 10, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, None) == -1   # stride too small
    assert lib.vark_compact_kv(p, p, 1 << 20, 1, 1, 4, 7, 12, sides, p, p, p, p, p, p, None) == -2
    assert lib.vark_build_offsets(p, 1, 4, 7, sides, 1, 64, None, p, p, p, None) == -1
    assert lib.vark_build_offsets(p, 1, 4, 7, sides, 1, 64, ctypes.c_void_p(20), p, p, p, None) == -3


@pytest.mark.parametrize("sides,L,H", [(SIDES_TINY, 3, 4), (SIDES_1024, 8, 32)])
def test_cache_size_accounting_matches_oracle(sides, L, H):
    keep = np.random.default_rng(L + H).integers(0, 2, size=(L, H, len(sides))).astype(np.uint8)
    got = vark.vark_cache_size_after_layer(keep, sides, 4, 128)
    assert np.array_equal(got, oracle.cache_size_after_layer(keep, sides, 4, 128))


def test_rank_stability_matches_oracle():
    rng = np.random.default_rng(5)
    for sides, L, H in ((SIDES_TINY, 2, 3), (SIDES_1024, 32, 16)):
        S = len(sides)
        a = rng.uniform(size=(L, H, S))
        b = np.round(a + 0.05 * rng.standard_normal(size=a.shape), 2)
        for budget in (5000, 1000):
            try:
                ref = oracle.rank_stability(a, b, sides, budget, 2)
            except oracle.BudgetError:
                continue
            got = vark.vark_rank_stability(a, b, sides, budget, 2)
            assert abs(got[0] - ref[0]) < 1e-12 and got[1] == ref[1]


@pytest.mark.parametrize("sides,L,H,budget", [(SIDES_TINY, 2, 3, 2500), (SIDES_1024, 32, 16, 1000),
                                               (SIDES_1024, 8, 32, 400)])
def test_early_pruning_schedule_matches_oracle(sides, L, H, budget):
    scas = np.round(np.random.default_rng(L * H).uniform(size=(L, H, len(sides))), 3)
    p_ref, e_ref = oracle.early_pruning_schedule(scas, sides, budget, 2)
    p_got, e_got = vark.vark_build_early_pruning_schedule(scas, sides, budget, 2)
    assert np.array_equal(p_got, p_ref) and np.array_equal(e_got, e_ref)


def test_generation_and_int8_calls_reject_bad_arguments_before_the_device():
    lib = vark.library()
    sides = (ctypes.c_int32 * 7)(*SIDES_TINY)
    p = ctypes.c_void_p(16)
    odd = ctypes.c_void_p(24)          # 8-byte but not 16-byte aligned
    # quantising compaction: k, v, layer_stride, L, B, H, S, D, sides, keep, head_off, seg_off, layer_base, kq, vq, ka, va
    assert lib.vark_quantize_kv_int8(None, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -1
    assert lib.vark_quantize_kv_int8(p, p, 1 << 20, 1, 1, 4, 7, 60, sides, p, p, p, p, p, p, p, p, None) == -2
    assert lib.vark_quantize_kv_int8(p, p, 1 << 20, 1, 1, 4, 7, 1024, sides, p, p, p, p, p, p, p, p, None) == -2
    assert lib.vark_quantize_kv_int8(p, p, 1 << 20, 1, 1, 4096, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -2
    assert lib.vark_quantize_kv_int8(p, p, 100, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -1
    assert lib.vark_quantize_kv_int8(p, p, (1 << 20) + 4, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -3
    assert lib.vark_quantize_kv_int8(p, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, odd, p, p, p, None) == -3
    # dequantisation: kq, vq, ka, va, kc_rows, B, H, S, D, sides, head_off, seg_off, kc, vc
    assert lib.vark_dequantize_layer_int8(None, p, p, p, 8, 1, 4, 7, 64, sides, p, p, p, p, None) == -1
    assert lib.vark_dequantize_layer_int8(p, p, p, p, 8, 1, 4, 7, 60, sides, p, p, p, p, None) == -2
    assert lib.vark_dequantize_layer_int8(p, p, p, p, 9, 2, 4, 7, 64, sides, p, p, p, p, None) == -2
    assert lib.vark_dequantize_layer_int8(p, p, p, p, 8, 1, 4, 7, 64, sides, p, p, odd, p, None) == -3
    assert lib.vark_dequantize_layer_int8(ctypes.c_void_p(20), p, p, p, 8, 1, 4, 7, 64, sides, p, p, p, p,
                                          None) == -3
    # append of one scale: scale outside the list
    assert lib.vark_append_scale(p, p, 1 << 20, 1, 1, 4, 7, 64, sides, 7, p, p, p, p, p, p, None) == -1
    # re-compaction: the source and destination must differ; max_scale within [0, S]
    assert lib.vark_recompact_kv(p, p, p, p, p, 1, 1, 4, 7, 64, sides, 3, p, p, p, p, p, p, None) == -1
    q = ctypes.c_void_p(4096)
    assert lib.vark_recompact_kv(p, p, p, p, p, 1, 1, 4, 7, 64, sides, 8, p, p, p, p, q, q, None) == -1
