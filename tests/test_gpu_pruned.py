"""GPU vs oracle: pruned-cache attention through the whole inference path
(offsets -> compaction -> pruned attention), edge cases included."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from synth import SIDES_TINY, SIDES_1024
from tests.helpers import Tables, bits_of, compact, dev_bf16, f64, pruned_layer

pytestmark = pytest.mark.gpu

O_ATOL = 2e-2


def _layer_inputs(sides, B, H, D, seed, with_bias, Tq=None):
    T = synth.n_tokens(sides)
    Tq = T if Tq is None else Tq
    qb = synth.normal_bf16_bits(synth.derive_key(70, seed, 0), (B, H, Tq, D))
    kb = synth.normal_bf16_bits(synth.derive_key(70, seed, 1), (B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(70, seed, 2), (B, H, T, D))
    tau = synth.gen_tau(seed, H)
    bias = synth.gen_bias(seed, H, len(sides)) if with_bias else None
    return qb, kb, vb, tau, bias


def _run(qb, kb, vb, keep, sides, tau, bias, query_scale):
    B, H, T, D = kb.shape
    tab = Tables(keep[None], sides, B, D)
    kd, vd = dev_bf16(kb), dev_bf16(vb)
    kc, vc = compact(kd[None], vd[None], tab, sides)
    out = pruned_layer(dev_bf16(qb), kc, vc, kd, vd, tab, 0, sides, query_scale, torch.from_numpy(tau).cuda(),
                       None if bias is None else torch.from_numpy(bias).cuda())
    return f64(bits_of(out))


@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("keep_kind", ["random", "all", "sinks_only", "none"])
def test_pruned_tiny_all_scales(with_bias, keep_kind):
    sides = SIDES_TINY
    B, H, D = 2, 4, 64
    qb, kb, vb, tau, bias = _layer_inputs(sides, B, H, D, 3, with_bias)
    S = len(sides)
    if keep_kind == "random":
        keep = np.random.default_rng(3).integers(0, 2, size=(H, S)).astype(np.uint8)
        keep[:, :2] = 1
    elif keep_kind == "all":
        keep = np.ones((H, S), dtype=np.uint8)
    elif keep_kind == "sinks_only":
        keep = np.zeros((H, S), dtype=np.uint8)
        keep[:, :2] = 1
    else:
        keep = np.zeros((H, S), dtype=np.uint8)   # empty compacted cache: local scale only
    O_gpu = _run(qb, kb, vb, keep, sides, tau, bias, -1)
    O_ref = oracle.pruned_attention(f64(qb), f64(kb), f64(vb), keep, sides, tau.astype(np.float64),
                                    None if bias is None else bias.astype(np.float64))
    assert np.abs(O_gpu - O_ref).max() <= O_ATOL
    if keep_kind == "all":
        O_full, _ = oracle.block_causal_attention(f64(qb), f64(kb), f64(vb), sides, tau.astype(np.float64),
                                                  None if bias is None else bias.astype(np.float64))
        assert np.abs(O_gpu - O_full).max() <= O_ATOL


@pytest.mark.parametrize("query_scale", [0, 3, 6])
def test_pruned_tiny_single_query_scale(query_scale):
    sides = SIDES_TINY
    g = oracle.ScaleGeometry(sides)
    B, H, D = 2, 3, 64
    qb, kb, vb, tau, bias = _layer_inputs(sides, B, H, D, 4, True, Tq=g.n[query_scale])
    keep = np.random.default_rng(4).integers(0, 2, size=(H, g.S)).astype(np.uint8)
    O_gpu = _run(qb, kb, vb, keep, sides, tau, bias, query_scale)
    O_ref = oracle.pruned_attention(f64(qb), f64(kb), f64(vb), keep, sides, tau.astype(np.float64),
                                    bias.astype(np.float64), query_scale=query_scale)
    assert np.abs(O_gpu - O_ref).max() <= O_ATOL


def test_pruned_1024_sampled_rows_all_scales():
    """1024^2 scale list, D=128, ragged keep per head, bias: sampled rows of
    every scale (first, last, tile boundaries, random) of every (b, h)."""
    sides = SIDES_1024
    g = oracle.ScaleGeometry(sides)
    B, H, D = 2, 4, 128
    qb, kb, vb, tau, bias = _layer_inputs(sides, B, H, D, 5, True)
    rng = np.random.default_rng(5)
    keep = rng.integers(0, 2, size=(H, g.S)).astype(np.uint8)
    keep[:, :2] = 1
    keep[0, :] = 1
    O_gpu = _run(qb, kb, vb, keep, sides, tau, bias, -1)
    for b in range(B):
        for h in range(H):
            kf, vf = f64(kb[b, h]), f64(vb[b, h])
            for kk in range(g.S):
                cand = [0, g.n[kk] - 1, 127, 128, int(rng.integers(g.n[kk]))]
                rows = np.unique([r for r in cand if r < g.n[kk]])
                o_ref = oatt_rows(f64(qb[b, h, g.off[kk] + rows]), kf, vf, keep[h], sides, kk, tau[h], bias[h])
                assert np.abs(O_gpu[b, h, g.off[kk] + rows] - o_ref).max() <= O_ATOL, (b, h, kk)


def test_pruned_1024_ten_heads_full():
    """1024^2 scales, 10 heads (the launch interleaves heads in groups of 8, so
    the last group is partial), ragged keep with a head that keeps nothing
    and one that keeps everything, bias: every output element of every scale
    against the oracle."""
    sides = SIDES_1024
    g = oracle.ScaleGeometry(sides)
    B, H, D = 1, 10, 128
    qb, kb, vb, tau, bias = _layer_inputs(sides, B, H, D, 15, True)
    keep = np.random.default_rng(15).integers(0, 2, size=(H, g.S)).astype(np.uint8)
    keep[:, :2] = 1
    keep[3, :] = 0
    keep[7, :] = 1
    O_gpu = _run(qb, kb, vb, keep, sides, tau, bias, -1)
    O_ref = oracle.pruned_attention(f64(qb), f64(kb), f64(vb), keep, sides, tau.astype(np.float64),
                                    bias.astype(np.float64))
    assert np.abs(O_gpu - O_ref).max() <= O_ATOL


def oatt_rows(q_rows, kf, vf, keep_h, sides, kk, tau_h, bias_h):
    from oracle.attention import pruned_attention_rows
    return pruned_attention_rows(q_rows, kf, vf, keep_h, sides, kk, float(tau_h),
                                 None if bias_h is None else np.asarray(bias_h, dtype=np.float64))


@pytest.mark.parametrize("budget_bp", [10000, 2000, 1000, 400])
@pytest.mark.parametrize("B", [1, 4, 16, 32])
def test_final_scale_sweep_sampled(budget_bp, B):
    """The 64x64 scale's 4,096 queries against the 10,521-token cache with
    seed-random retained sets per head (final-scale sweep), inputs made on the
    device at full size; sampled rows against the oracle."""
    w = synth.WORKLOADS["final_scale"]
    sides, H, D, kq = w.sides, w.heads, w.head_dim, w.query_scale
    g = oracle.ScaleGeometry(sides)
    T = g.T
    keep = synth.random_keep(synth.derive_key(w.base_seed, budget_bp), H, sides, budget_bp, w.n_sinks, kq)
    keys = [synth.derive_key(w.base_seed, 9, B, i) for i in range(3)]
    q = synth.normal_bf16_torch(keys[0], (B, H, g.n[kq], D), device="cuda")
    kd = synth.normal_bf16_torch(keys[1], (B, H, T, D), device="cuda")
    vd = synth.normal_bf16_torch(keys[2], (B, H, T, D), device="cuda")
    tau = synth.gen_tau(w.base_seed, H)
    tab = Tables(keep, sides, B, D)
    kc, vc = compact(kd[None], vd[None], tab, sides)
    out = pruned_layer(q, kc, vc, kd, vd, tab, 0, sides, kq, torch.from_numpy(tau).cuda(), None)
    rng = np.random.default_rng(budget_bp + B)
    pairs = {(B - 1, H - 1)} | {(int(rng.integers(B)), int(rng.integers(H))) for _ in range(5)}
    for b, h in sorted(pairs):
        rows = np.unique(np.concatenate([[0, 127, 128, g.n[kq] - 1], rng.integers(0, g.n[kq], size=4)]))
        kf = f64(synth.rows_bf16_bits(keys[1], (B, H, T, D), (b, h), 0, T))
        vf = f64(synth.rows_bf16_bits(keys[2], (B, H, T, D), (b, h), 0, T))
        qr = f64(synth.rows_bf16_bits(keys[0], (B, H, g.n[kq], D), (b, h), 0, g.n[kq]))[rows]
        o_ref = oatt_rows(qr, kf, vf, keep[0, h], sides, kq, tau[h], None)
        o_gpu = out[b, h, torch.from_numpy(rows).cuda()].float().cpu().numpy()
        assert np.abs(o_gpu - o_ref).max() <= O_ATOL, (b, h)
