"""Time-varying schedule on the GPU (BINARY-HEATKV with GREEDYEARLYPRUNING,
the library's reading): scale by scale, attention of scale k's queries over
the cache held after step k-1 plus scale k, then the cache moves to the
retained set of step k (re-compaction of survivors + append of scale k).
After every step the cache equals the oracle's compaction of that step's
retained set bit for bit; outputs match the oracle on samples and the
one-shot kernel bit for bit."""
import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from tests.helpers import Tables, bits_of, dev_bf16, f64, status_word

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sides,D,budget", [(synth.SIDES_TINY, 64, 3000), (synth.SIDES_1024, 128, 1500)])
def test_early_pruning_generation_loop(sides, D, budget):
    g = oracle.ScaleGeometry(sides)
    L, B, H, T, S = 2, 2, 4, g.T, g.S
    kb = synth.normal_bf16_bits(synth.derive_key(85, D, 1), (L, B, H, T, D))
    vb = synth.normal_bf16_bits(synth.derive_key(85, D, 2), (L, B, H, T, D))
    qb = synth.normal_bf16_bits(synth.derive_key(85, D, 3), (L, B, H, T, D))
    scas = synth.random_scas(D + budget, L, H, S)
    prefix, evict = vark.vark_build_early_pruning_schedule(scas, sides, budget, 2)
    p_ref, e_ref = oracle.early_pruning_schedule(scas, sides, budget, 2)
    assert np.array_equal(prefix, p_ref) and np.array_equal(evict, e_ref)
    assert prefix[-1] > 0                      # the budget forces evictions
    tau = [torch.from_numpy(synth.gen_tau(30 + l, H)).cuda() for l in range(L)]
    kd, vd, qd = dev_bf16(kb), dev_bf16(vb), dev_bf16(qb)
    st = status_word()
    cap = L * B * H * T * D
    bufs = [(torch.zeros(cap, dtype=torch.bfloat16, device="cuda"), torch.zeros(cap, dtype=torch.bfloat16, device="cuda"))
            for _ in range(2)]
    prev = None          # (tables, buffers) of the cache held after the previous step
    rng = np.random.default_rng(D)
    for k in range(S):
        sl = slice(g.off[k], g.off[k] + g.n[k])
        k_new, v_new = kd[:, :, :, sl].contiguous(), vd[:, :, :, sl].contiguous()
        keep_prev = oracle.keep_after_step(evict, k - 1) if k > 0 else np.zeros((L, H, S), dtype=np.uint8)
        tab_prev = prev[0] if prev else Tables(keep_prev, sides, B, D)
        kc_prev, vc_prev = prev[1] if prev else bufs[1]
        for l in range(L):
            q_k = qd[l][:, :, sl].contiguous()
            out = torch.empty_like(q_k)
            base, rows = tab_prev.elem_base(l), tab_prev.kc_rows(l)
            vark.vark_pruned_attention_step(q_k, kc_prev[base:base + rows * D] if rows else None,
                                            vc_prev[base:base + rows * D] if rows else None, rows, k_new[l],
                                            v_new[l], sides, k, tab_prev.head_off[l], tab_prev.seg_off[l],
                                            tab_prev.past_len[l], tau[l], None, out, st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            b, h = int(rng.integers(B)), int(rng.integers(H))
            rows_s = np.unique([0, g.n[k] - 1, int(rng.integers(g.n[k]))])
            o_ref = oracle.pruned_attention_rows(f64(qb[l, b, h, g.off[k] + rows_s]), f64(kb[l, b, h]),
                                                 f64(vb[l, b, h]), keep_prev[l, h], sides, k, float(tau[l][h].item()))
            got = f64(bits_of(out[b, h, torch.from_numpy(rows_s).cuda()]))
            assert np.abs(got - o_ref).max() <= 2e-2, (k, l)
        # move to the retained set of step k
        keep_k = oracle.keep_after_step(evict, k)
        tab_k = Tables(keep_k, sides, B, D)
        kc_k, vc_k = bufs[k % 2]
        vark.vark_recompact_kv(kc_prev, vc_prev, tab_prev.head_off, tab_prev.seg_off, tab_prev.layer_base, L, B, H,
                               sides, D, k, tab_k.keep, tab_k.head_off, tab_k.seg_off, tab_k.layer_base, kc_k, vc_k)
        vark.vark_append_scale(k_new, v_new, B * H * g.n[k] * D, L, B, H, sides, D, k, tab_k.keep, tab_k.head_off,
                               tab_k.seg_off, tab_k.layer_base, kc_k, vc_k)
        torch.cuda.synchronize()
        ho, so, pl, lb = oracle.build_offsets(keep_k, sides, B, D)
        kref, vref = oracle.compact_kv(kb, vb, keep_k, sides, ho, so, lb)
        assert np.array_equal(bits_of(kc_k)[:tab_k.total], kref), k
        assert np.array_equal(bits_of(vc_k)[:tab_k.total], vref), k
        # the absolute budget holds once the schedule can meet it
        held = int((keep_k * np.array(g.n)[None, None, :]).sum())
        if prefix[k] < L * H:
            assert held * 10000 <= budget * L * H * T
        prev = (tab_k, (kc_k, vc_k))
