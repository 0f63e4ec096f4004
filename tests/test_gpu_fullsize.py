"""Full-size GPU runs of the multi-layer workloads, in the launch
configurations the benchmark times, checked on samples against the oracle:

* 32 layers x 16 heads, batch 8, 10% (pruned inference) and 8 layers x 32
  heads, batch 4, 4% (larger-model shape): schedule (host, bit-exact),
  offsets (bit-exact), one compaction launch over all layers (sampled blocks
  bit-exact against the generator), pruned attention of sampled layers
  (sampled rows of every query scale against the oracle);
* the calibration launch of the larger shape (8 seeds x 32 heads): mass sums
  to one and sampled masses / output rows against the oracle;
* the int8 / 4-bit / 3-bit quantising compaction of the 32-layer workload:
  sampled blocks' codes and scales, and one layer's dequantisation, bit-exact.

Inputs are made on the device by the host-reproducible generator; schedules
come from synthetic S-CAS so no oracle input comes from the CUDA path."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from tests.helpers import Tables, bits_of, check_status, f64, pruned_layer, status_word

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
O_ATOL = 2e-2


def _pipeline(wname):
    w = synth.WORKLOADS[wname]
    sides, L, H, D, B = w.sides, w.layers, w.heads, w.head_dim, w.batch
    g = oracle.ScaleGeometry(sides)
    T = g.T
    scas = synth.random_scas(w.base_seed, L, H, g.S)
    keep = vark.vark_build_schedule(scas, sides, w.budget_bp, w.n_sinks)
    assert np.array_equal(keep, oracle.build_schedule(scas, sides, w.budget_bp, w.n_sinks))
    tab = Tables(keep, sides, B, D)
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    torch.cuda.synchronize()
    assert np.array_equal(tab.head_off.cpu().numpy(), ho) and np.array_equal(tab.seg_off.cpu().numpy(), so)
    assert np.array_equal(tab.past_len.cpu().numpy(), pl) and np.array_equal(tab.layer_base.cpu().numpy(), lb)
    kkey, vkey = synth.qkv_key(w, 0, "k", "infer"), synth.qkv_key(w, 0, "v", "infer")
    shape = (L, B, H, T, D)
    kd = synth.normal_bf16_torch(kkey, shape, device="cuda")
    vd = synth.normal_bf16_torch(vkey, shape, device="cuda")
    kc = torch.empty(max(tab.total, 8), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    vark.vark_compact_kv(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off,
                         tab.layer_base, kc, vc)
    torch.cuda.synchronize()
    rng = np.random.default_rng(L * 1000 + H)
    # compaction: sampled (layer, batch, head) blocks, every kept scale, bit-exact
    for _ in range(6):
        l, b, h = int(rng.integers(L)), int(rng.integers(B)), int(rng.integers(H))
        R_l = int(lb[l + 1] - lb[l]) // (B * D)
        for s in range(g.S):
            if not keep[l, h, s]:
                continue
            row = int(lb[l]) // D + b * R_l + int(ho[l, h]) + int(so[l, h, s])
            got_k = bits_of(kc[row * D:(row + g.n[s]) * D].view(g.n[s], D))
            got_v = bits_of(vc[row * D:(row + g.n[s]) * D].view(g.n[s], D))
            assert np.array_equal(got_k, synth.rows_bf16_bits(kkey, shape, (l, b, h), g.off[s], g.off[s] + g.n[s]))
            assert np.array_equal(got_v, synth.rows_bf16_bits(vkey, shape, (l, b, h), g.off[s], g.off[s] + g.n[s]))
    # pruned attention of sampled layers, all query scales
    for l in sorted({0, L // 2, L - 1}):
        qkey = synth.qkv_key(w, l, "q", "infer")
        qshape = (B, H, T, D)
        q = synth.normal_bf16_torch(qkey, qshape, device="cuda")
        tau = synth.gen_tau(synth.layer_seed(w, l), H)
        bias = synth.gen_bias(synth.layer_seed(w, l), H, g.S) if w.with_bias else None
        out = pruned_layer(q, kc, vc, kd[l], vd[l], tab, l, sides, -1, torch.from_numpy(tau).cuda(),
                           None if bias is None else torch.from_numpy(bias).cuda())
        for _ in range(4):
            b, h = int(rng.integers(B)), int(rng.integers(H))
            kf = f64(synth.rows_bf16_bits(kkey, shape, (l, b, h), 0, T))
            vf = f64(synth.rows_bf16_bits(vkey, shape, (l, b, h), 0, T))
            for kk in range(g.S):
                rows = np.unique([0, g.n[kk] - 1, min(128, g.n[kk] - 1), int(rng.integers(g.n[kk]))])
                qr = f64(synth.rows_bf16_bits(qkey, qshape, (b, h), g.off[kk], g.L[kk]))[rows]
                o_ref = oracle.pruned_attention_rows(qr, kf, vf, keep[l, h], sides, kk, float(tau[h]),
                                                     None if bias is None else bias[h].astype(np.float64))
                o_gpu = out[b, h, g.off[kk] + torch.from_numpy(rows).cuda()].float().cpu().numpy()
                assert np.abs(o_gpu - o_ref).max() <= O_ATOL, (l, b, h, kk)
        del q, out


def test_pruned_inference_32_layers_full_size():
    _pipeline("pruned_32l")


def test_larger_model_8_layers_32_heads_full_size():
    _pipeline("large_8l")


def test_larger_model_calibration_launch_full_size():
    w = synth.WORKLOADS["large_8l"]
    sides, H, D, Bc = w.sides, w.heads, w.head_dim, w.n_seeds
    g = oracle.ScaleGeometry(sides)
    T, S = g.T, g.S
    keys = [synth.qkv_key(w, 0, x, "calib") for x in ("q", "k", "v")]
    shape = (Bc, H, T, D)
    q, k, v = (synth.normal_bf16_torch(key, shape, device="cuda") for key in keys)
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
    h = 29
    acc = np.zeros((S, 8))
    for b in range(Bc):
        qb, kb, vb = (f64(synth.rows_bf16_bits(key, shape, (b, h), 0, g.L[7])) for key in keys)
        for kk in range(8):
            _, m = oracle.attention_rows(qb[g.off[kk]:g.L[kk]], kb, vb, sides, kk, float(tau[h]),
                                         bias[h].astype(np.float64))
            acc[:, kk] += m.sum(axis=0) / (Bc * g.n[kk])
    np.testing.assert_allclose(M[h, :, :8], acc, rtol=1e-3)
    b, kk = Bc - 1, 12
    rows = np.array([0, 127, 128, 4095])
    kb, vb = (f64(synth.rows_bf16_bits(key, shape, (b, h), 0, T)) for key in keys[1:])
    qb = f64(synth.rows_bf16_bits(keys[0], shape, (b, h), g.off[kk], g.L[kk]))[rows]
    o_ref, _ = oracle.attention_rows(qb, kb, vb, sides, kk, float(tau[h]), bias[h].astype(np.float64))
    o_gpu = out[b, h, g.off[kk] + torch.from_numpy(rows).cuda()].float().cpu().numpy()
    assert np.abs(o_gpu - o_ref).max() <= O_ATOL


@pytest.mark.parametrize("bits", [8, 4, 3])
def test_quantised_cache_full_size(bits):
    """The quantising compaction of all 32 layers of the pruned-inference
    workload (batch 8, 16 heads, 10%) in one call, as the benchmark runs it:
    sampled (layer, batch, head) blocks, every kept scale, codes and scales
    bit-exact against the oracle on the generator's rows; then one sampled
    layer dequantised, sampled rows bit-exact."""
    w = synth.WORKLOADS["pruned_32l"]
    sides, L, H, D, B = w.sides, w.layers, w.heads, w.head_dim, w.batch
    g = oracle.ScaleGeometry(sides)
    T = g.T
    scas = synth.random_scas(w.base_seed, L, H, g.S)
    keep = vark.vark_build_schedule(scas, sides, w.budget_bp, w.n_sinks)
    tab = Tables(keep, sides, B, D)
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kkey, vkey = synth.qkv_key(w, 0, "k", "infer"), synth.qkv_key(w, 0, "v", "infer")
    shape = (L, B, H, T, D)
    kd = synth.normal_bf16_torch(kkey, shape, device="cuda")
    vd = synth.normal_bf16_torch(vkey, shape, device="cuda")
    total = tab.total
    num, den = {8: (1, 1), 4: (1, 2), 3: (3, 8)}[bits]
    kq = torch.zeros(max(num * total // den, 16), dtype=torch.uint8 if bits != 8 else torch.int8, device="cuda")
    vq = torch.zeros_like(kq)
    tdt = torch.float32 if bits == 8 else torch.int16
    ks = torch.zeros((L, B, H, g.S, D), dtype=tdt, device="cuda")
    vs = torch.zeros_like(ks)
    fn = {8: vark.vark_quantize_kv_int8, 4: vark.vark_quantize_kv_int4, 3: vark.vark_quantize_kv_int3}[bits]
    fn(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off, tab.layer_base, kq, vq, ks, vs)
    torch.cuda.synchronize()
    quant = {8: oracle.quantize_block, 4: oracle.quantize_block_int4, 3: oracle.quantize_block_int3}[bits]
    unpack = {8: lambda a, D: a.view(np.int8).reshape(-1, D), 4: oracle.unpack_int4, 3: oracle.unpack_int3}[bits]
    deq = {8: oracle.dequantize_block, 4: oracle.dequantize_block_int4, 3: oracle.dequantize_block_int3}[bits]

    def table(x, l, b, h, s):
        t = x[l, b, h, s].cpu().numpy()
        return t if bits == 8 else t.view(np.uint16)

    rng = np.random.default_rng(91 + bits)
    kqh = kq.cpu().numpy().view(np.uint8)
    vqh = vq.cpu().numpy().view(np.uint8)
    for _ in range(6):
        l, b, h = int(rng.integers(L)), int(rng.integers(B)), int(rng.integers(H))
        R_l = int(lb[l + 1] - lb[l]) // (B * D)
        for s in range(g.S):
            if not keep[l, h, s]:
                continue
            e0 = int(lb[l]) + (b * R_l + int(ho[l, h]) + int(so[l, h, s])) * D
            lo, hi = num * e0 // den, num * (e0 + g.n[s] * D) // den
            for src, key, x in ((kqh, kkey, ks), (vqh, vkey, vs)):
                rows = synth.rows_bf16_bits(key, shape, (l, b, h), g.off[s], g.off[s] + g.n[s])
                codes, scale = quant(rows)
                assert np.array_equal(unpack(src[lo:hi], D), codes), (bits, l, b, h, s)
                assert np.array_equal(table(x, l, b, h, s), scale), (bits, l, b, h, s)
    # one layer's dequantisation, sampled (batch, head) rows
    l = int(rng.integers(L))
    rows_l = int(lb[l + 1] - lb[l]) // D
    kc = torch.zeros(max(rows_l * D, 16), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    base = num * int(lb[l]) // den
    dfn = {8: vark.vark_dequantize_layer_int8, 4: vark.vark_dequantize_layer_int4,
           3: vark.vark_dequantize_layer_int3}[bits]
    dfn(kq[base:], vq[base:], ks[l], vs[l], rows_l, B, H, sides, D, tab.head_off[l], tab.seg_off[l], kc, vc)
    torch.cuda.synchronize()
    R_l = rows_l // B
    kch = bits_of(kc)[:rows_l * D].reshape(rows_l, D)
    for _ in range(4):
        b, h = int(rng.integers(B)), int(rng.integers(H))
        for s in range(g.S):
            if not keep[l, h, s]:
                continue
            r0 = b * R_l + int(ho[l, h]) + int(so[l, h, s])
            codes, scale = quant(synth.rows_bf16_bits(kkey, shape, (l, b, h), g.off[s], g.off[s] + g.n[s]))
            assert np.array_equal(kch[r0:r0 + g.n[s]], deq(codes, scale)), (bits, l, b, h, s)
    del kd, vd, kq, vq, ks, vs, kc, vc
    torch.cuda.empty_cache()
