"""The seeded input generator: CPU/torch agreement, moments, workload sets."""
import numpy as np
import torch

import synth


def test_numpy_and_torch_generators_agree_bitwise():
    key = synth.derive_key(7, 1, 2)
    a = synth.normal_bf16_bits(key, (2, 3, 155, 64))
    b = synth.normal_bf16_torch(key, (2, 3, 155, 64), chunk=1 << 12).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(a, b)
    idx = np.array([0, 1, 12345, a.size - 1], dtype=np.uint64)
    assert np.array_equal(synth.normal_bf16_bits_at(key, idx), a.ravel()[idx.astype(np.int64)])


def test_generator_rows_helper():
    key = synth.derive_key(3)
    shape = (2, 3, 50, 16)
    full = synth.normal_bf16_bits(key, shape)
    assert np.array_equal(synth.rows_bf16_bits(key, shape, (1, 2), 10, 30), full[1, 2, 10:30])


def test_generator_moments_and_rounding():
    bits = synth.normal_bf16_bits(synth.derive_key(11), (1 << 18,))
    x = synth.bf16_bits_to_f32(bits).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert np.abs(x).max() <= 6.0
    # bf16 round-to-nearest-even on hand-checked values
    v = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0000002], dtype=np.float32)
    r = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(v))
    assert list(r) == [1.0, 1.0, 1.015625, -2.5, 3.0]


def test_tau_and_bias_ranges():
    tau = synth.gen_tau(3, 16)
    assert tau.dtype == np.float32 and np.all((tau >= 0.5) & (tau <= 2.0))
    bias = synth.gen_bias(3, 16, 13)
    nz = (bias != 0).sum(axis=1)
    assert np.all((nz >= 1) & (nz <= 3)) and np.all((bias >= 0) & (bias <= 2))


def test_random_keep_sets_meet_budget():
    sides = synth.SIDES_1024
    n = np.array([s * s for s in sides])
    for budget in (10000, 2000, 1000, 400):
        keep = synth.random_keep(5, 16, sides, budget, 2, 12)
        assert np.all(keep[0, :, :2] == 1) and np.all(keep[0, :, 12] == 1)
        past = (keep[0, :, :12] * n[None, :12]).sum(axis=1)
        assert np.all(past * 10000 <= budget * n.sum())
        if budget == 10000:
            assert np.all(keep == 1)
