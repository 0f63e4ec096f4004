"""Quantised retained cache on the GPU: int8 codes and per-(block, channel)
absmax bit-exact with the oracle, per-layer dequantisation bit-exact, and
pruned attention over the dequantised cache against the oracle run on the same
values (past scales dequantised, the local scale from the dense cache)."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from tests.helpers import Tables, bits_of, dev_bf16, f64, status_word

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sides,D", [(synth.SIDES_TINY, 64), (synth.SIDES_1024, 128)])
def test_int8_cache_bit_exact_and_attention(sides, D):
    g = oracle.ScaleGeometry(sides)
    L, B, H, T, S = 2, 2, 3, g.T, g.S
    kb = synth.normal_bf16_bits(synth.derive_key(95, D, 1), (L, B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(95, D, 2), (L, B, H, T, D))
    qb = synth.normal_bf16_bits(synth.derive_key(95, D, 3), (B, H, T, D))
    keep = np.random.default_rng(D).integers(0, 2, size=(L, H, S)).astype(np.uint8)
    keep[:, :, :2] = 1
    tab = Tables(keep, sides, B, D)
    kd, vd = dev_bf16(kb), dev_bf16(vb)
    kq = torch.empty(max(tab.total, 16), dtype=torch.int8, device="cuda")
    vq = torch.empty_like(kq)
    ka = torch.empty((L, B, H, S, D), dtype=torch.float32, device="cuda")
    va = torch.empty_like(ka)
    vark.vark_quantize_kv_int8(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off,
                               tab.layer_base, kq, vq, ka, va)
    torch.cuda.synchronize()
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kq_ref, vq_ref, ka_ref, va_ref = oracle.quantize_kv(kb, vb, keep, sides, ho, so, lb)
    assert np.array_equal(kq.cpu().numpy()[:tab.total], kq_ref)
    assert np.array_equal(vq.cpu().numpy()[:tab.total], vq_ref)
    assert np.array_equal(ka.cpu().numpy(), ka_ref) and np.array_equal(va.cpu().numpy(), va_ref)
    tau = torch.from_numpy(synth.gen_tau(96, H)).cuda()
    st = status_word()
    for l in range(L):
        rows = tab.kc_rows(l)
        base = tab.elem_base(l)
        kc = torch.empty(max(rows * D, 16), dtype=torch.bfloat16, device="cuda")
        vc = torch.empty_like(kc)
        vark.vark_dequantize_layer_int8(kq[base:], vq[base:], ka[l], va[l], rows, B, H, sides, D, tab.head_off[l],
                                        tab.seg_off[l], kc, vc)
        torch.cuda.synchronize()
        # dequantised values of every kept block, bit-exact
        deq_k = np.array(kb[l], copy=True)
        deq_v = np.array(vb[l], copy=True)
        R_l = rows // B
        kcb, vcb = bits_of(kc)[:rows * D].reshape(-1, D), bits_of(vc)[:rows * D].reshape(-1, D)
        for b in range(B):
            for h in range(H):
                for s in range(S):
                    if not keep[l, h, s]:
                        continue
                    sl = slice(g.off[s], g.off[s] + g.n[s])
                    rk = oracle.dequantize_block(kq_ref[int(lb[l]):][(b * R_l + ho[l, h] + so[l, h, s]) * D:][:g.n[s] * D]
                                                 .reshape(g.n[s], D), ka_ref[l, b, h, s])
                    rv = oracle.dequantize_block(vq_ref[int(lb[l]):][(b * R_l + ho[l, h] + so[l, h, s]) * D:][:g.n[s] * D]
                                                 .reshape(g.n[s], D), va_ref[l, b, h, s])
                    r0 = b * R_l + ho[l, h] + so[l, h, s]
                    assert np.array_equal(kcb[r0:r0 + g.n[s]], rk) and np.array_equal(vcb[r0:r0 + g.n[s]], rv)
                    deq_k[b, h, sl], deq_v[b, h, sl] = rk, rv
        # pruned attention over the dequantised past + dense local scale
        out = torch.empty((B, H, T, D), dtype=torch.bfloat16, device="cuda")
        q = dev_bf16(qb)
        vark.vark_pruned_attention(q, kc if rows else None, vc if rows else None, rows, kd[l], vd[l], sides, -1,
                                   tab.head_off[l], tab.seg_off[l], tab.past_len[l], tau, None, out, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        O = f64(bits_of(out))
        for b in range(B):
            for h in range(H):
                for kk in range(S):
                    k_eff, v_eff = f64(deq_k[b, h]), f64(deq_v[b, h])
                    loc = slice(g.off[kk], g.off[kk] + g.n[kk])
                    k_eff[loc], v_eff[loc] = f64(kb[l, b, h, loc]), f64(vb[l, b, h, loc])
                    rows_s = np.unique([0, g.n[kk] - 1])
                    o_ref = oracle.pruned_attention_rows(f64(qb[b, h, g.off[kk] + rows_s]), k_eff, v_eff, keep[l, h],
                                                         sides, kk, float(tau[h].item()))
                    assert np.abs(O[b, h, g.off[kk] + rows_s] - o_ref).max() <= 2e-2, (l, b, h, kk)


def _expected_layer_bf16(q_ref, a_ref, keep_l, g, ho_l, so_l, lb_l, R_l, B, H, D):
    """The oracle's dequantised compacted block of one layer, [B * R_l][D] bf16 bits."""
    out = np.zeros((B * R_l, D), dtype=np.uint16)
    for b in range(B):
        for h in range(H):
            for s in range(g.S):
                if not keep_l[h, s]:
                    continue
                r0 = b * R_l + int(ho_l[h]) + int(so_l[h, s])
                codes = q_ref[lb_l + r0 * D:lb_l + (r0 + g.n[s]) * D].reshape(g.n[s], D)
                out[r0:r0 + g.n[s]] = oracle.dequantize_block(codes, a_ref[b, h, s])
    return out


@pytest.mark.parametrize("sides,D,L,B,H,mode", [
    (synth.SIDES_TINY, 96, 2, 3, 5, "random"),          # 12 vectors per row: a ragged thread layout
    (synth.SIDES_1024, 256, 1, 2, 2, "all"),            # every block, the 4096-row one split over the cluster
    (synth.SIDES_1024, 128, 2, 1, 3, "sparse"),         # a layer with nothing kept, a head with nothing kept
    (synth.SIDES_TINY, 64, 3, 1, 1024, "random"),       # several (layer, head) launch groups
    (synth.SIDES_1024, 8, 1, 2, 4, "random"),           # one vector per row
])
def test_int8_codes_and_dequant_bit_exact_shapes(sides, D, L, B, H, mode):
    g = oracle.ScaleGeometry(sides)
    T, S = g.T, g.S
    kb = synth.normal_bf16_bits(synth.derive_key(97, D, H), (L, B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(98, D, H), (L, B, H, T, D))
    rng = np.random.default_rng(D * 7 + H)
    if mode == "all":
        keep = np.ones((L, H, S), dtype=np.uint8)
    else:
        keep = rng.integers(0, 2, size=(L, H, S)).astype(np.uint8)
    if mode == "sparse":
        keep[0] = 0
        keep[1, 1] = 0
        keep[1, 0, -1] = 1
    tab = Tables(keep, sides, B, D)
    kd, vd = dev_bf16(kb), dev_bf16(vb)
    kq = torch.full((max(tab.total, 16),), 77, dtype=torch.int8, device="cuda")
    vq = torch.full_like(kq, 77)
    ka = torch.full((L, B, H, S, D), 5.0, dtype=torch.float32, device="cuda")
    va = torch.full_like(ka, 5.0)
    vark.vark_quantize_kv_int8(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off,
                               tab.layer_base, kq, vq, ka, va)
    torch.cuda.synchronize()
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kq_ref, vq_ref, ka_ref, va_ref = oracle.quantize_kv(kb, vb, keep, sides, ho, so, lb)
    assert np.array_equal(kq.cpu().numpy()[:tab.total], kq_ref)
    assert np.array_equal(vq.cpu().numpy()[:tab.total], vq_ref)
    assert np.array_equal(ka.cpu().numpy(), ka_ref) and np.array_equal(va.cpu().numpy(), va_ref)
    for l in range(L):
        rows = tab.kc_rows(l)
        base = tab.elem_base(l)
        kc = torch.zeros(max(rows * D, 16), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        vark.vark_dequantize_layer_int8(kq[base:], vq[base:], ka[l], va[l], rows, B, H, sides, D, tab.head_off[l],
                                        tab.seg_off[l], kc, vc)
        torch.cuda.synchronize()
        R_l = rows // B
        ek = _expected_layer_bf16(kq_ref, ka_ref[l], keep[l], g, ho[l], so[l], int(lb[l]), R_l, B, H, D)
        ev = _expected_layer_bf16(vq_ref, va_ref[l], keep[l], g, ho[l], so[l], int(lb[l]), R_l, B, H, D)
        assert np.array_equal(bits_of(kc)[:rows * D].reshape(-1, D), ek), l
        assert np.array_equal(bits_of(vc)[:rows * D].reshape(-1, D), ev), l
