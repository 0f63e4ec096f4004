"""3-bit quantised retained cache on the GPU: packed codes and per-(block,
channel) bf16 scales bit-exact with the oracle over a sweep of shapes, and the
per-layer dequantisation bit-exact."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from tests.helpers import Tables, bits_of, dev_bf16

pytestmark = pytest.mark.gpu


def _expected_layer_bf16(q_ref, s_ref, keep_l, g, ho_l, so_l, lb_l, R_l, B, H, D):
    """The oracle's dequantised compacted block of one layer, [B * R_l][D] bf16 bits."""
    out = np.zeros((B * R_l, D), dtype=np.uint16)
    for b in range(B):
        for h in range(H):
            for s in range(g.S):
                if not keep_l[h, s]:
                    continue
                r0 = b * R_l + int(ho_l[h]) + int(so_l[h, s])
                lo = 3 * (lb_l + r0 * D) // 8
                codes = oracle.unpack_int3(q_ref[lo:lo + 3 * g.n[s] * D // 8], D)
                out[r0:r0 + g.n[s]] = oracle.dequantize_block_int3(codes, s_ref[b, h, s])
    return out


@pytest.mark.parametrize("sides,D,L,B,H,mode", [
    (synth.SIDES_TINY, 64, 2, 2, 3, "random"),
    (synth.SIDES_TINY, 96, 2, 3, 5, "random"),          # 12 vectors per row: a ragged thread layout
    (synth.SIDES_1024, 128, 1, 2, 2, "all"),            # every block, the 4096-row one split over the cluster
    (synth.SIDES_1024, 128, 2, 1, 3, "sparse"),         # a layer with nothing kept, a head with nothing kept
    (synth.SIDES_TINY, 64, 3, 1, 1024, "random"),       # several (layer, head) launch groups
    (synth.SIDES_1024, 8, 1, 2, 4, "random"),           # one vector per row
])
def test_int3_codes_and_dequant_bit_exact_shapes(sides, D, L, B, H, mode):
    g = oracle.ScaleGeometry(sides)
    T, S = g.T, g.S
    kb = synth.normal_bf16_bits(synth.derive_key(297, D, H), (L, B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(298, D, H), (L, B, H, T, D))
    rng = np.random.default_rng(D * 13 + H)
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
    nbytes = max(3 * tab.total // 8, 16)
    kq = torch.full((nbytes,), 0x5A, dtype=torch.uint8, device="cuda")
    vq = torch.full_like(kq, 0x5A)
    ks = torch.full((L, B, H, S, D), 7, dtype=torch.int16, device="cuda")
    vs = torch.full_like(ks, 7)
    vark.vark_quantize_kv_int3(kd, vd, B * H * T * D, L, B, H, sides, D, tab.keep, tab.head_off, tab.seg_off,
                               tab.layer_base, kq, vq, ks, vs)
    torch.cuda.synchronize()
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kq_ref, vq_ref, ks_ref, vs_ref = oracle.quantize_kv_int3(kb, vb, keep, sides, ho, so, lb)
    assert np.array_equal(kq.cpu().numpy()[:3 * tab.total // 8], kq_ref)
    assert np.array_equal(vq.cpu().numpy()[:3 * tab.total // 8], vq_ref)
    assert np.array_equal(ks.cpu().numpy().view(np.uint16), ks_ref)
    assert np.array_equal(vs.cpu().numpy().view(np.uint16), vs_ref)
    for l in range(L):
        rows = tab.kc_rows(l)
        base = 3 * tab.elem_base(l) // 8
        kc = torch.zeros(max(rows * D, 16), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        vark.vark_dequantize_layer_int3(kq[base:], vq[base:], ks[l], vs[l], rows, B, H, sides, D, tab.head_off[l],
                                        tab.seg_off[l], kc, vc)
        torch.cuda.synchronize()
        R_l = rows // B
        ek = _expected_layer_bf16(kq_ref, ks_ref[l], keep[l], g, ho[l], so[l], int(lb[l]), R_l, B, H, D)
        ev = _expected_layer_bf16(vq_ref, vs_ref[l], keep[l], g, ho[l], so[l], int(lb[l]), R_l, B, H, D)
        assert np.array_equal(bits_of(kc)[:rows * D].reshape(-1, D), ek), l
        assert np.array_equal(bits_of(vc)[:rows * D].reshape(-1, D), ev), l

