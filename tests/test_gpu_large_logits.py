"""GPU vs oracle with logits far outside the range of N(0,1) inputs: a few
query rows and key rows are scaled up (values still exact bf16, used by both
sides), so some logits reach a few hundred and the online softmax meets
large running-max jumps, row maxima dominated by one key, and probabilities
that underflow to zero."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from synth import SIDES_TINY, SIDES_1024
from tests.helpers import Tables, bits_of, check_status, compact, dev_bf16, f64, pruned_layer, status_word

pytestmark = pytest.mark.gpu
O_ATOL = 2e-2


def _scaled_bits(key, shape, rows_every, factor):
    x = synth.bf16_bits_to_f32(synth.normal_bf16_bits(key, shape)).copy()
    x[..., ::rows_every, :] *= np.float32(factor)
    return synth.f32_to_bf16_bits(x)


def _inputs(sides, B, H, D, seed):
    T = synth.n_tokens(sides)
    qb = _scaled_bits(synth.derive_key(80, seed, 0), (B, H, T, D), 7, 6.0)
    kb = _scaled_bits(synth.derive_key(80, seed, 1), (B, H, T, D), 5, 4.0)
    vb = synth.normal_bf16_bits(synth.derive_key(80, seed, 2), (B, H, T, D))
    tau = np.full(H, 2.0, dtype=np.float32)
    bias = synth.gen_bias(seed, H, len(sides))
    return qb, kb, vb, tau, bias


@pytest.mark.parametrize("sides,D", [(SIDES_TINY, 64), (SIDES_1024, 128)])
def test_calibration_with_large_logits(sides, D):
    B, H = 1, 2
    qb, kb, vb, tau, bias = _inputs(sides, B, H, D, 1 + D)
    x = float(tau[0]) * np.abs(f64(qb[0, 0]) @ f64(kb[0, 0]).T).max() / np.sqrt(D)
    assert x > 100.0
    S = len(sides)
    q, k, v = dev_bf16(qb), dev_bf16(kb), dev_bf16(vb)
    mass = torch.zeros((H, S, S), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    st = status_word()
    vark.vark_scas_accumulate(q, k, v, sides, torch.from_numpy(tau).cuda(), torch.from_numpy(bias).cuda(), mass,
                              out, st)
    check_status(st)
    O_ref, m = oracle.block_causal_attention(f64(qb), f64(kb), f64(vb), sides, tau.astype(np.float64),
                                             bias.astype(np.float64))
    assert np.abs(f64(bits_of(out)) - O_ref).max() <= O_ATOL
    np.testing.assert_allclose(mass.cpu().numpy().astype(np.float64), oracle.scas_mass(m, sides), rtol=1e-3)


def test_pruned_attention_with_large_logits():
    sides = SIDES_TINY
    B, H, D = 2, 3, 64
    qb, kb, vb, tau, bias = _inputs(sides, B, H, D, 9)
    keep = np.random.default_rng(9).integers(0, 2, size=(H, len(sides))).astype(np.uint8)
    keep[:, :2] = 1
    tab = Tables(keep[None], sides, B, D)
    kd, vd = dev_bf16(kb), dev_bf16(vb)
    kc, vc = compact(kd[None], vd[None], tab, sides)
    out = pruned_layer(dev_bf16(qb), kc, vc, kd, vd, tab, 0, sides, -1, torch.from_numpy(tau).cuda(),
                       torch.from_numpy(bias).cuda())
    O_ref = oracle.pruned_attention(f64(qb), f64(kb), f64(vb), keep, sides, tau.astype(np.float64),
                                    bias.astype(np.float64))
    assert np.abs(f64(bits_of(out)) - O_ref).max() <= O_ATOL


def test_calibration_max_jump_in_a_later_full_tile():
    """One key of the last 1024^2 scale (row 8,000: key tile 62, a full tile of
    a single scale) is set to 2 in every channel and the queries of that scale
    are shifted by +0.5, so nearly every one of them meets its row maximum
    only there, above the running max of the earlier tiles by more than the
    rescale threshold (a few rows stay below it, so a warp mixes both cases):
    those rows must rescale and recompute the columns they had already
    exponentiated against the old maximum."""
    sides = SIDES_1024
    B, H, D = 1, 1, 128
    T = synth.n_tokens(sides)
    g = oracle.ScaleGeometry(sides)
    qf = synth.bf16_bits_to_f32(synth.normal_bf16_bits(synth.derive_key(81, 0), (B, H, T, D))).copy()
    qf[0, 0, g.off[12]:] += np.float32(0.5)
    qb = synth.f32_to_bf16_bits(qf)
    kf = synth.bf16_bits_to_f32(synth.normal_bf16_bits(synth.derive_key(81, 1), (B, H, T, D))).copy()
    kf[0, 0, 8000] = np.float32(2.0)
    kb = synth.f32_to_bf16_bits(kf)
    vb = synth.normal_bf16_bits(synth.derive_key(81, 2), (B, H, T, D))
    tau = np.full(H, 1.5, dtype=np.float32)
    bias = np.zeros((H, len(sides)), dtype=np.float32)
    assert g.off[12] <= 62 * 128 and 63 * 128 <= g.off[12] + g.n[12] and 62 * 128 <= 8000 < 63 * 128
    logits = float(tau[0]) * (f64(qb[0, 0, g.off[12]:]) @ f64(kb[0, 0]).T) / np.sqrt(D)
    jump = (logits[:, 8000] - logits[:, :62 * 128].max(axis=1)) * np.log2(np.e)
    assert 0.9 < (jump > 8.0).mean() < 1.0    # nearly every row of scale 12 crosses the rescale threshold at tile 62
    S = len(sides)
    q, k, v = dev_bf16(qb), dev_bf16(kb), dev_bf16(vb)
    mass = torch.zeros((H, S, S), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    st = status_word()
    vark.vark_scas_accumulate(q, k, v, sides, torch.from_numpy(tau).cuda(), torch.from_numpy(bias).cuda(), mass,
                              out, st)
    check_status(st)
    O_ref, m = oracle.block_causal_attention(f64(qb), f64(kb), f64(vb), sides, tau.astype(np.float64),
                                             bias.astype(np.float64))
    assert np.abs(f64(bits_of(out)) - O_ref).max() <= O_ATOL
    np.testing.assert_allclose(mass.cpu().numpy().astype(np.float64), oracle.scas_mass(m, sides), rtol=1e-3)
