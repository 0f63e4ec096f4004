"""Generation order on the GPU: for each scale k, pruned attention of scale
k's queries over the cache appended so far plus scale k itself, then the
append of scale k.  It must reproduce the one-shot path (compaction of the
finished cache, then pruned attention of every scale) bit for bit -- outputs of
every scale and the final compacted cache -- and match the oracle on samples;
the cache-size accounting must end at the compacted layout's size."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from tests.helpers import Tables, bits_of, compact, dev_bf16, f64, status_word

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sides,D,with_bias", [(synth.SIDES_TINY, 64, False), (synth.SIDES_1024, 128, True)])
def test_generation_loop_matches_one_shot_bit_exact(sides, D, with_bias):
    g = oracle.ScaleGeometry(sides)
    L, B, H, T, S = 2, 2, 4, g.T, g.S
    kb = synth.normal_bf16_bits(synth.derive_key(80, D, 1), (L, B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(80, D, 2), (L, B, H, T, D))
    qb = synth.normal_bf16_bits(synth.derive_key(80, D, 3), (L, B, H, T, D))
    keep = np.random.default_rng(D).integers(0, 2, size=(L, H, S)).astype(np.uint8)
    keep[:, :, :2] = 1
    keep[0, 1, :] = 0
    tau = [torch.from_numpy(synth.gen_tau(10 + l, H)).cuda() for l in range(L)]
    bias = [torch.from_numpy(synth.gen_bias(10 + l, H, S)).cuda() if with_bias else None for l in range(L)]
    kd, vd, qd = dev_bf16(kb), dev_bf16(vb), dev_bf16(qb)
    tab = Tables(keep, sides, B, D)
    st = status_word()

    # one shot
    kc1, vc1 = compact(kd, vd, tab, sides)
    outs1 = []
    for l in range(L):
        out = torch.empty_like(qd[l])
        base, rows = tab.elem_base(l), tab.kc_rows(l)
        vark.vark_pruned_attention(qd[l], kc1[base:base + rows * D] if rows else None,
                                   vc1[base:base + rows * D] if rows else None, rows, kd[l], vd[l], sides, -1,
                                   tab.head_off[l], tab.seg_off[l], tab.past_len[l], tau[l], bias[l], out, st)
        outs1.append(out)

    # generation order
    kc2 = torch.zeros_like(kc1)
    vc2 = torch.zeros_like(vc1)
    for k in range(S):
        sl = slice(g.off[k], g.off[k] + g.n[k])
        k_new = kd[:, :, :, sl].contiguous()
        v_new = vd[:, :, :, sl].contiguous()
        for l in range(L):
            q_k = qd[l][:, :, sl].contiguous()
            out_k = torch.empty_like(q_k)
            base, rows = tab.elem_base(l), tab.kc_rows(l)
            vark.vark_pruned_attention_step(q_k, kc2[base:base + rows * D] if rows else None,
                                            vc2[base:base + rows * D] if rows else None, rows, k_new[l], v_new[l],
                                            sides, k, tab.head_off[l], tab.seg_off[l], tab.past_len[l], tau[l],
                                            bias[l], out_k, st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            assert np.array_equal(bits_of(out_k), bits_of(outs1[l][:, :, sl].contiguous())), (k, l)
        vark.vark_append_scale(k_new, v_new, B * H * g.n[k] * D, L, B, H, sides, D, k, tab.keep, tab.head_off,
                               tab.seg_off, tab.layer_base, kc2, vc2)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(kc2), bits_of(kc1)) and np.array_equal(bits_of(vc2), bits_of(vc1))

    # oracle on samples of the generation-order outputs (= one-shot outputs)
    rng = np.random.default_rng(1)
    for _ in range(4):
        l, b, h, k = int(rng.integers(L)), int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(S))
        rows = np.unique([0, g.n[k] - 1, int(rng.integers(g.n[k]))])
        o_ref = oracle.pruned_attention_rows(f64(qb[l, b, h, g.off[k] + rows]), f64(kb[l, b, h]), f64(vb[l, b, h]),
                                             keep[l, h], sides, k, float(tau[l][h].item()),
                                             None if bias[l] is None else bias[l][h].cpu().numpy().astype(np.float64))
        got = f64(bits_of(outs1[l][b, h, torch.from_numpy(g.off[k] + rows).cuda()]))
        assert np.abs(got - o_ref).max() <= 2e-2

    # cache-size accounting ends at the compacted layout's size (K and V, 2 bytes)
    sz = vark.vark_cache_size_after_layer(keep, sides, B, D)
    assert sz[-1, -1] == 4 * tab.total
