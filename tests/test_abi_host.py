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


def _no_device():
    """True when no CUDA device is visible: calls that pass every host check
    with placeholder pointers are made only then (on a GPU they would launch)."""
    import torch
    return not torch.cuda.is_available()


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


def test_size_limits_are_status_codes():
    """Shapes whose arithmetic would overflow, or whose calibration tiles would
    not fit in shared memory, are refused before any array is read or any
    device call is made."""
    lib = vark.library()
    p = ctypes.c_void_p(16)
    # calibration at D = 128: 30 scales fit the shared memory, 31 do not (D = 64: 32 fit)
    s31 = (ctypes.c_int32 * 31)(*([1] * 31))
    s30 = (ctypes.c_int32 * 30)(*([1] * 30))
    s32 = (ctypes.c_int32 * 32)(*([1] * 32))
    assert lib.vark_scas_accumulate(p, p, p, 1, 4, 128, 31, s31, p, None, p, None, p, None) == -2
    if _no_device():   # these pass the shape checks and stop at the device check
        assert lib.vark_scas_accumulate(p, p, p, 1, 4, 128, 30, s30, p, None, p, None, p, None) in (-7, -5)
        assert lib.vark_scas_accumulate(p, p, p, 1, 4, 64, 32, s32, p, None, p, None, p, None) in (-7, -5)
    # schedule budget arithmetic: F = L * H * T tokens with F * 10000 < 2^63.  32 scales of side
    # 4096 give T = 2^29; L * H = 2^20 makes F = 2^49 (fits), 2^21 makes 2^50 > 9.2e14.  The
    # arrays passed are tiny: a refused shape must not read them.
    big = (ctypes.c_int32 * 32)(*([4096] * 32))
    tiny = np.zeros(8)
    keep = np.zeros(8, dtype=np.uint8)
    assert lib.vark_build_schedule(tiny.ctypes.data, 1 << 11, 1 << 10, 32, big, 5000, 2, keep.ctypes.data) == -2
    assert lib.vark_rank_stability(tiny.ctypes.data, tiny.ctypes.data, 1 << 11, 1 << 10, 32, big, 5000, 2,
                                   ctypes.byref(ctypes.c_double()), ctypes.byref(ctypes.c_double())) == -2
    pre = np.zeros(32, dtype=np.int32)
    assert lib.vark_build_early_pruning_schedule(tiny.ctypes.data, 1 << 11, 1 << 10, 32, big, 5000, 2,
                                                 pre.ctypes.data, keep.ctypes.data) == -2
    out = np.zeros(8, dtype=np.int64)
    assert lib.vark_cache_size_after_layer(keep.ctypes.data, 1 << 16, 1 << 10, 32, big, 1 << 10, 128,
                                           out.ctypes.data) == -2
    # the same builder at a small size still works
    sc = np.random.default_rng(3).uniform(size=(2, 3, 7))
    assert np.array_equal(vark.vark_build_schedule(sc, SIDES_TINY, 5000, 2), oracle.build_schedule(sc, SIDES_TINY,
                                                                                                   5000, 2))


def test_binding_refuses_mismatched_tensor_sizes():
    """Every wrapper compares its tensors with the shape it hands to the C call
    and raises ValueError before a pointer is taken (CPU tensors here: the size
    check comes first, so nothing reaches the library)."""
    import torch
    sides = SIDES_TINY
    S, T, D, B, H = 7, 155, 64, 2, 4
    bf = torch.bfloat16
    f32 = torch.float32
    i32 = torch.int32
    q = torch.zeros((B, H, T, D), dtype=bf)
    st = torch.zeros(1, dtype=i32)
    tau, bias, mass = torch.zeros(H), torch.zeros(H, S), torch.zeros(H, S, S)
    good = dict(q=q, k=q, v=q, sides=sides, tau=tau, bias=bias, mass=mass, out=q, dev_status=st)
    for key, bad in (("q", torch.zeros((B, H, T - 1, D), dtype=bf)), ("k", torch.zeros((B, H, T, 32), dtype=bf)),
                     ("v", torch.zeros((B + 1, H, T, D), dtype=bf)), ("out", torch.zeros((B, H, T, D + 8), dtype=bf)),
                     ("tau", torch.zeros(H - 1)), ("bias", torch.zeros(H, S - 1)), ("mass", torch.zeros(H, S, S - 1))):
        with pytest.raises(ValueError):
            vark.vark_scas_accumulate(**{**good, key: bad})
    with pytest.raises(TypeError):          # sizes right: the device check is what refuses a CPU tensor
        vark.vark_scas_accumulate(**good)
    L = 2
    keep = torch.ones((L, H, S), dtype=torch.uint8)
    tabs = dict(head_off=torch.zeros(L, H, dtype=i32), seg_off=torch.zeros(L, H, S, dtype=i32),
                past_len=torch.zeros(L, H, S, dtype=i32), layer_base=torch.zeros(L + 1, dtype=torch.int64))
    for key in tabs:
        bad = torch.zeros(tabs[key].numel() + 1, dtype=tabs[key].dtype)
        with pytest.raises(ValueError):
            vark.vark_build_offsets(keep, sides, B, D, **{**tabs, key: bad})
    kd = torch.zeros((L, B, H, T, D), dtype=bf)
    comp = dict(k=kd, v=kd, layer_stride=B * H * T * D, L=L, B=B, H=H, sides=sides, D=D, keep=keep,
                head_off=tabs["head_off"], seg_off=tabs["seg_off"], layer_base=tabs["layer_base"], kc=kd, vc=kd)
    for key, bad in (("k", kd[:1]), ("layer_stride", B * H * T * D - 8), ("keep", keep[:1]),
                     ("seg_off", tabs["seg_off"][:1])):
        with pytest.raises(ValueError):
            vark.vark_compact_kv(**{**comp, key: bad})
    # pruned attention: one layer, every query scale
    pr = dict(q=q, kc=torch.zeros(B * 10 * D, dtype=bf), vc=torch.zeros(B * 10 * D, dtype=bf), kc_rows=B * 10,
              k_dense=q, v_dense=q, sides=sides, query_scale=-1, head_off=torch.zeros(H, dtype=i32),
              seg_off=torch.zeros(H, S, dtype=i32), past_len=torch.zeros(H, S, dtype=i32), tau=tau, bias=bias,
              out=q, dev_status=st)
    for key, bad in (("q", torch.zeros((B, H, 64, D), dtype=bf)), ("kc", torch.zeros(B * 10 * D - 1, dtype=bf)),
                     ("kc_rows", B * 10 + 1), ("out", q[:1]), ("head_off", torch.zeros(H + 1, dtype=i32)),
                     ("past_len", torch.zeros(H, dtype=i32)), ("query_scale", S)):
        with pytest.raises(ValueError):
            vark.vark_pruned_attention(**{**pr, key: bad})
    q6 = torch.zeros((B, H, 64, D), dtype=bf)
    with pytest.raises(TypeError):          # query scale 6 (64 rows): sizes right
        vark.vark_pruned_attention(**{**pr, "q": q6, "out": q6, "query_scale": 6})
    step = {**pr, "q": q6, "out": q6, "scale": 6}
    step.pop("query_scale")
    step["k_local"] = step.pop("k_dense")
    step["v_local"] = step.pop("v_dense")
    with pytest.raises(ValueError):         # k_local must hold the scale's rows only
        vark.vark_pruned_attention_step(**step)
    with pytest.raises(ValueError):
        vark.vark_dequantize_layer_int8(torch.zeros(10, dtype=torch.int8), torch.zeros(10, dtype=torch.int8),
                                        torch.zeros(B * H * S * D), torch.zeros(B * H * S * D), 2, 1, H, sides, D,
                                        torch.zeros(H, dtype=i32), torch.zeros(H, S, dtype=i32),
                                        torch.zeros(2 * D, dtype=bf), torch.zeros(2 * D, dtype=bf))


def test_int4_calls_reject_bad_arguments_before_the_device():
    lib = vark.library()
    sides = (ctypes.c_int32 * 7)(*SIDES_TINY)
    p = ctypes.c_void_p(16)
    odd = ctypes.c_void_p(24)           # 8-byte but not 16-byte aligned
    two = ctypes.c_void_p(18)           # 2-byte aligned only
    # quantising compaction: k, v, layer_stride, L, B, H, S, D, sides, keep, head_off, seg_off, layer_base, kq, vq, ks, vs
    assert lib.vark_quantize_kv_int4(None, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -1
    assert lib.vark_quantize_kv_int4(p, p, 1 << 20, 1, 1, 4, 7, 60, sides, p, p, p, p, p, p, p, p, None) == -2
    assert lib.vark_quantize_kv_int4(p, p, 100, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -1
    assert lib.vark_quantize_kv_int4(p, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, odd, p, p, p, None) == -3
    assert lib.vark_quantize_kv_int4(p, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, odd, p, None) == -3
    # dequantisation: kq, vq, ks, vs, kc_rows, B, H, S, D, sides, head_off, seg_off, kc, vc (codes 4-byte aligned)
    assert lib.vark_dequantize_layer_int4(None, p, p, p, 8, 1, 4, 7, 64, sides, p, p, p, p, None) == -1
    assert lib.vark_dequantize_layer_int4(p, p, p, p, 9, 2, 4, 7, 64, sides, p, p, p, p, None) == -2
    assert lib.vark_dequantize_layer_int4(two, p, p, p, 8, 1, 4, 7, 64, sides, p, p, p, p, None) == -3
    # 4-byte aligned codes pass the checks; kc_rows = 0 returns before any launch
    assert lib.vark_dequantize_layer_int4(ctypes.c_void_p(20), p, p, p, 0, 1, 4, 7, 64, sides, p, p, p, p,
                                          None) in (-7, -5, 0)


def test_int3_calls_reject_bad_arguments_before_the_device():
    lib = vark.library()
    sides = (ctypes.c_int32 * 7)(*SIDES_TINY)
    p = ctypes.c_void_p(16)
    odd = ctypes.c_void_p(24)           # 8-byte but not 16-byte aligned
    assert lib.vark_quantize_kv_int3(None, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -1
    assert lib.vark_quantize_kv_int3(p, p, 1 << 20, 1, 1, 4, 7, 60, sides, p, p, p, p, p, p, p, p, None) == -2
    assert lib.vark_quantize_kv_int3(p, p, 100, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, p, p, None) == -1
    assert lib.vark_quantize_kv_int3(p, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, odd, p, p, p, None) == -3
    assert lib.vark_quantize_kv_int3(p, p, 1 << 20, 1, 1, 4, 7, 64, sides, p, p, p, p, p, p, odd, p, None) == -3
    assert lib.vark_dequantize_layer_int3(None, p, p, p, 8, 1, 4, 7, 64, sides, p, p, p, p, None) == -1
    assert lib.vark_dequantize_layer_int3(p, p, p, p, 9, 2, 4, 7, 64, sides, p, p, p, p, None) == -2
    assert lib.vark_dequantize_layer_int3(p, p, odd, p, 8, 1, 4, 7, 64, sides, p, p, p, p, None) == -3
    # 3-byte groups need no alignment: an odd code pointer passes; kc_rows = 0 returns before any launch
    assert lib.vark_dequantize_layer_int3(ctypes.c_void_p(17), p, p, p, 0, 1, 4, 7, 64, sides, p, p, p, p,
                                          None) in (-7, -5, 0)


def test_packed_attention_calls_reject_bad_arguments_before_the_device():
    lib = vark.library()
    sides = (ctypes.c_int32 * 7)(*SIDES_TINY)
    p = ctypes.c_void_p(16)
    odd = ctypes.c_void_p(24)           # 8-byte but not 16-byte aligned

    def call(bits, q=p, kq=p, tab=p, kc_rows=8, B=1, D=64, qs=-1, dense=p):
        fn = getattr(lib, f"vark_pruned_attention_int{bits}")
        return fn(q, kq, p, tab, p, kc_rows, dense, p, B, 4, 7, D, sides, qs, p, p, p, p, None, p, p, None)

    for bits in (8, 4, 3):
        D = 128 if bits == 3 else 64
        assert call(bits, q=None, D=D) == -1
        assert call(bits, kq=None, D=D) == -1          # codes required when a past exists
        assert call(bits, D=D, qs=7) == -1             # query scale out of range
        assert call(bits, D=D, kc_rows=9, B=2) == -2   # rows not a multiple of the batch
        assert call(bits, D=96) == -2                  # head_dim 64 or 128 only
        assert call(bits, kq=odd, D=D) == -3           # whole tiles are bulk-copied: 16-byte codes
        assert call(bits, tab=odd, D=D) == -3
        assert call(bits, dense=odd, D=D) == -3
    # 3-bit rows of D = 64 are 24 bytes: not a multiple of 16, refused
    assert call(3, D=64) == -2
    if _no_device():   # these pass every host check and stop at the device check
        for bits in (8, 4, 3):
            assert call(bits, D=128) in (-7, -5)
            assert call(bits, kq=None, kc_rows=0, D=128) in (-7, -5)   # no past: codes may be absent


def test_binding_refuses_mismatched_packed_attention_sizes():
    """The attention-over-codes wrappers check codes, tables and the usual
    query / table sizes before any pointer is taken (CPU tensors)."""
    import torch
    sides = SIDES_TINY
    S, T, D, B, H, rows = 7, 155, 64, 2, 4, 20
    bf, i32 = torch.bfloat16, torch.int32
    q = torch.zeros((B, H, T, D), dtype=bf)
    base = dict(q=q, kc_rows=rows, k_dense=q, v_dense=q, sides=sides, query_scale=-1,
                head_off=torch.zeros(H, dtype=i32), seg_off=torch.zeros(H, S, dtype=i32),
                past_len=torch.zeros(H, S, dtype=i32), tau=torch.zeros(H), bias=torch.zeros(H, S), out=q,
                dev_status=torch.zeros(1, dtype=i32))
    cases = {
        8: (vark.vark_pruned_attention_int8, "k_absmax", "v_absmax", torch.int8, torch.float32, rows * D),
        4: (vark.vark_pruned_attention_int4, "k_scale", "v_scale", torch.uint8, torch.int16, rows * D // 2),
        3: (vark.vark_pruned_attention_int3, "k_scale", "v_scale", torch.uint8, torch.int16, rows * 3 * D // 8),
    }
    for bits, (fn, kt, vt, code_t, tab_t, nbytes) in cases.items():
        good = {**base, "kq": torch.zeros(nbytes, dtype=code_t), "vq": torch.zeros(nbytes, dtype=code_t),
                kt: torch.zeros(B * H * S * D, dtype=tab_t), vt: torch.zeros(B * H * S * D, dtype=tab_t)}
        for key, bad in (("kq", torch.zeros(nbytes - 1, dtype=code_t)), ("vq", torch.zeros(nbytes - 1, dtype=code_t)),
                         (kt, torch.zeros(B * H * S * D - 1, dtype=tab_t)), ("kc_rows", rows + 1),
                         ("q", torch.zeros((B, H, T - 1, D), dtype=bf)), ("past_len", torch.zeros(H, dtype=i32)),
                         ("query_scale", S)):
            with pytest.raises(ValueError):
                fn(**{**good, key: bad})
        with pytest.raises(TypeError):      # sizes right: the device check refuses a CPU tensor
            fn(**good)
