"""Pruned attention straight over a quantised retained cache, the past
dequantised inside the attention kernel (vark_pruned_attention_int8 / _int4 /
_int3): its output equals, bit for bit, the separate path (per-layer
dequantisation into a bf16 block, then vark_pruned_attention over it), and
sampled rows match the oracle's pruned attention over the oracle's
dequantised values.  The 1024^2 scale list gives heads whose pasts span many
key tiles next to heads with none; the tiny list gives pasts of one tile."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from tests.helpers import Tables, bits_of, dev_bf16, f64, status_word

pytestmark = pytest.mark.gpu

# bits -> (quantise, dequantise one layer, fused attention, code dtype, table dtype, code bytes per element)
_CALLS = {
    8: (vark.vark_quantize_kv_int8, vark.vark_dequantize_layer_int8, vark.vark_pruned_attention_int8,
        torch.int8, torch.float32, (1, 1)),
    4: (vark.vark_quantize_kv_int4, vark.vark_dequantize_layer_int4, vark.vark_pruned_attention_int4,
        torch.uint8, torch.int16, (1, 2)),
    3: (vark.vark_quantize_kv_int3, vark.vark_dequantize_layer_int3, vark.vark_pruned_attention_int3,
        torch.uint8, torch.int16, (3, 8)),
}


def _oracle_block(bits, q_ref, t_ref, e0, n, D):
    """The oracle's dequantised block of n rows whose first element is e0."""
    if bits == 8:
        return oracle.dequantize_block(q_ref[e0:e0 + n * D].reshape(n, D), t_ref)
    if bits == 4:
        return oracle.dequantize_block_int4(oracle.unpack_int4(q_ref[e0 // 2:(e0 + n * D) // 2], D), t_ref)
    return oracle.dequantize_block_int3(oracle.unpack_int3(q_ref[3 * e0 // 8:3 * (e0 + n * D) // 8], D), t_ref)


def _oracle_quantize(bits, kb, vb, keep, sides, ho, so, lb):
    fn = {8: oracle.quantize_kv, 4: oracle.quantize_kv_int4, 3: oracle.quantize_kv_int3}[bits]
    return fn(kb, vb, keep, sides, ho, so, lb)


@pytest.mark.parametrize("bits,sides,D,B,H,mode", [
    (8, synth.SIDES_TINY, 64, 2, 3, "random"),
    (4, synth.SIDES_TINY, 64, 2, 3, "random"),
    (3, synth.SIDES_TINY, 128, 2, 3, "random"),
    (8, synth.SIDES_1024, 128, 2, 2, "random"),    # one staging slot (16 KB code tiles)
    (4, synth.SIDES_1024, 128, 2, 2, "random"),
    (3, synth.SIDES_1024, 128, 2, 2, "random"),
    (4, synth.SIDES_1024, 64, 1, 3, "all"),         # every scale kept: the longest pasts
])
def test_packed_past_attention(bits, sides, D, B, H, mode):
    quantize, dequantize, fused, code_t, tab_t, (num, den) = _CALLS[bits]
    g = oracle.ScaleGeometry(sides)
    L, T, S = 2, g.T, g.S
    key = 400 + bits
    kb = synth.normal_bf16_bits(synth.derive_key(key, D, 1), (L, B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(key, D, 2), (L, B, H, T, D))
    qb = synth.normal_bf16_bits(synth.derive_key(key, D, 3), (L, B, H, T, D))
    if mode == "all":
        keep = np.ones((L, H, S), dtype=np.uint8)
    else:
        keep = np.random.default_rng(bits * 7 + D).integers(0, 2, size=(L, H, S)).astype(np.uint8)
        keep[:, :, :2] = 1
        keep[1, 0, 2:] = 0      # a head whose past is the two sink scales only
    tab = Tables(keep, sides, B, D)
    kd, vd, qd = dev_bf16(kb), dev_bf16(vb), dev_bf16(qb)
    nbytes = max(num * tab.total // den, 16)
    kq = torch.empty(nbytes, dtype=code_t, device="cuda")
    vq = torch.empty_like(kq)
    kt = torch.empty((L, B, H, S, D), dtype=tab_t, device="cuda")
    vt = torch.empty_like(kt)
    quantize(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off, tab.layer_base,
             kq, vq, kt, vt)
    torch.cuda.synchronize()
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kq_ref, vq_ref, kt_ref, vt_ref = _oracle_quantize(bits, kb, vb, keep, sides, ho, so, lb)
    tau = torch.from_numpy(synth.gen_tau(key, H)).cuda()
    bias = torch.from_numpy(synth.gen_bias(key, H, S)).cuda()
    for l in range(L):
        rows = tab.kc_rows(l)
        b0 = num * tab.elem_base(l) // den
        st = status_word()
        # separate path: the layer's bf16 block, then attention over it
        kc = torch.zeros(max(rows * D, 16), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        dequantize(kq[b0:], vq[b0:], kt[l], vt[l], rows, B, H, sides, D, tab.head_off[l], tab.seg_off[l], kc, vc)
        out_sep = torch.empty_like(qd[l])
        vark.vark_pruned_attention(qd[l], kc if rows else None, vc if rows else None, rows, kd[l], vd[l], sides,
                                   -1, tab.head_off[l], tab.seg_off[l], tab.past_len[l], tau, bias, out_sep, st)
        # fused path
        out = torch.full_like(qd[l], float("nan"))
        fused(qd[l], kq[b0:], vq[b0:], kt[l], vt[l], rows, kd[l], vd[l], sides, -1, tab.head_off[l],
              tab.seg_off[l], tab.past_len[l], tau, bias, out, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, vark.vark_status_string(int(st.item()))
        O = bits_of(out)
        assert np.array_equal(O, bits_of(out_sep)), l
        # sampled rows against the oracle over its own dequantised past
        Of = f64(O)
        R_l = rows // B
        for b in range(B):
            for h in range(H):
                k_eff, v_eff = f64(kb[l, b, h]), f64(vb[l, b, h])
                for s in range(S):
                    if keep[l, h, s]:
                        sl = slice(g.off[s], g.off[s] + g.n[s])
                        e0 = int(lb[l]) + (b * R_l + int(ho[l, h]) + int(so[l, h, s])) * D
                        k_eff[sl] = f64(_oracle_block(bits, kq_ref, kt_ref[l, b, h, s], e0, g.n[s], D))
                        v_eff[sl] = f64(_oracle_block(bits, vq_ref, vt_ref[l, b, h, s], e0, g.n[s], D))
                for kk in range(S):
                    ke, ve = k_eff.copy(), v_eff.copy()
                    loc = slice(g.off[kk], g.off[kk] + g.n[kk])
                    ke[loc], ve[loc] = f64(kb[l, b, h, loc]), f64(vb[l, b, h, loc])   # local scale: dense
                    rs = np.unique([0, min(127, g.n[kk] - 1), min(128, g.n[kk] - 1), g.n[kk] - 1])
                    ref = oracle.pruned_attention_rows(f64(qb[l, b, h, g.off[kk] + rs]), ke, ve, keep[l, h], sides,
                                                       kk, float(tau[h].item()), bias.cpu().numpy()[h])
                    assert np.abs(Of[b, h, g.off[kk] + rs] - ref).max() <= 2e-2, (l, b, h, kk)


def test_packed_past_final_scale_query_batch():
    """The final scale's queries alone (query_scale = S - 1) at batch 8 over a
    4-bit past: every CTA of a head converts the same long past."""
    quantize, dequantize, fused, code_t, tab_t, (num, den) = _CALLS[4]
    sides, D, B, H = synth.SIDES_1024, 128, 8, 2
    g = oracle.ScaleGeometry(sides)
    L, T, S = 1, g.T, g.S
    kb = synth.normal_bf16_bits(synth.derive_key(431, D, 1), (L, B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(431, D, 2), (L, B, H, T, D))
    qb = synth.normal_bf16_bits(synth.derive_key(431, D, 3), (B, H, g.n[-1], D))
    keep = np.zeros((L, H, S), dtype=np.uint8)
    keep[:, :, :2] = 1
    keep[0, 0, [6, 9, 11, 12]] = 1
    keep[0, 1, [4, 10, 12]] = 1
    tab = Tables(keep, sides, B, D)
    kd, vd, qd = dev_bf16(kb), dev_bf16(vb), dev_bf16(qb)
    kq = torch.empty(max(num * tab.total // den, 16), dtype=code_t, device="cuda")
    vq = torch.empty_like(kq)
    kt = torch.empty((L, B, H, S, D), dtype=tab_t, device="cuda")
    vt = torch.empty_like(kt)
    quantize(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off, tab.layer_base,
             kq, vq, kt, vt)
    rows = tab.kc_rows(0)
    tau = torch.from_numpy(synth.gen_tau(432, H)).cuda()
    st = status_word()
    kc = torch.zeros(rows * D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    dequantize(kq, vq, kt[0], vt[0], rows, B, H, sides, D, tab.head_off[0], tab.seg_off[0], kc, vc)
    out_sep = torch.empty_like(qd)
    vark.vark_pruned_attention(qd, kc, vc, rows, kd[0], vd[0], sides, S - 1, tab.head_off[0], tab.seg_off[0],
                               tab.past_len[0], tau, None, out_sep, st)
    out = torch.full_like(qd, float("nan"))
    fused(qd, kq, vq, kt[0], vt[0], rows, kd[0], vd[0], sides, S - 1, tab.head_off[0], tab.seg_off[0],
          tab.past_len[0], tau, None, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, vark.vark_status_string(int(st.item()))
    assert np.array_equal(bits_of(out), bits_of(out_sep))


def _scaled_bf16_bits(bits, e):
    """bf16 bits of x * 2^e (round to nearest even; subnormal results kept)."""
    f = (f64(bits) * 2.0 ** e).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


@pytest.mark.parametrize("bits,D", [(8, 64), (4, 64), (4, 128), (3, 128)])
def test_packed_past_subnormal_scales(bits, D):
    """K and V of magnitude ~2^-128, so every scale and most dequantised values
    are subnormal: the in-kernel expansion must still equal the dequantiser."""
    quantize, dequantize, fused, code_t, tab_t, (num, den) = _CALLS[bits]
    sides, B, H = synth.SIDES_TINY, 2, 2
    g = oracle.ScaleGeometry(sides)
    L, T, S = 1, g.T, g.S
    kb = _scaled_bf16_bits(synth.normal_bf16_bits(synth.derive_key(441, D, 1), (L, B, H, T, D)), -128)
    vb = _scaled_bf16_bits(synth.normal_bf16_bits(synth.derive_key(441, D, 2), (L, B, H, T, D)), -128)
    qb = synth.normal_bf16_bits(synth.derive_key(441, D, 3), (B, H, T, D))
    keep = np.ones((L, H, S), dtype=np.uint8)
    tab = Tables(keep, sides, B, D)
    kd, vd, qd = dev_bf16(kb), dev_bf16(vb), dev_bf16(qb)
    kq = torch.empty(max(num * tab.total // den, 16), dtype=code_t, device="cuda")
    vq = torch.empty_like(kq)
    kt = torch.empty((L, B, H, S, D), dtype=tab_t, device="cuda")
    vt = torch.empty_like(kt)
    quantize(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off, tab.layer_base,
             kq, vq, kt, vt)
    rows = tab.kc_rows(0)
    tau = torch.from_numpy(synth.gen_tau(442, H)).cuda()
    st = status_word()
    kc = torch.zeros(rows * D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    dequantize(kq, vq, kt[0], vt[0], rows, B, H, sides, D, tab.head_off[0], tab.seg_off[0], kc, vc)
    out_sep = torch.empty_like(qd)
    vark.vark_pruned_attention(qd, kc, vc, rows, kd[0], vd[0], sides, -1, tab.head_off[0], tab.seg_off[0],
                               tab.past_len[0], tau, None, out_sep, st)
    out = torch.full_like(qd, float("nan"))
    fused(qd, kq, vq, kt[0], vt[0], rows, kd[0], vd[0], sides, -1, tab.head_off[0], tab.seg_off[0],
          tab.past_len[0], tau, None, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, vark.vark_status_string(int(st.item()))
    vals = f64(bits_of(vc)[:rows * D])
    assert np.any((vals != 0) & (np.abs(vals) < 2.0 ** -126))   # the case is really subnormal
    assert np.array_equal(bits_of(out), bits_of(out_sep))
