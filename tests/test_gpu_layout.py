"""GPU vs oracle, bit-exact: offset tables and cache compaction."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import SIDES_TINY, SIDES_1024
from tests.helpers import Tables, bits_of, compact, dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sides,L,H,B,D,seed", [
    (SIDES_TINY, 1, 4, 1, 64, 0), (SIDES_TINY, 3, 5, 2, 64, 1), (SIDES_1024, 32, 16, 8, 128, 2),
    (SIDES_1024, 8, 32, 4, 128, 3), (SIDES_1024, 2, 3, 1, 128, 4)])
def test_offsets_bit_exact(sides, L, H, B, D, seed):
    rng = np.random.default_rng(seed)
    keep = rng.integers(0, 2, size=(L, H, len(sides))).astype(np.uint8)
    keep[0, 0, :] = 0          # a head that keeps nothing
    if H > 1:
        keep[0, 1, :] = 1      # a head that keeps everything
    tab = Tables(keep, sides, B, D)
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    torch.cuda.synchronize()
    assert np.array_equal(tab.head_off.cpu().numpy(), ho)
    assert np.array_equal(tab.seg_off.cpu().numpy(), so)
    assert np.array_equal(tab.past_len.cpu().numpy(), pl)
    assert np.array_equal(tab.layer_base.cpu().numpy(), lb)


@pytest.mark.parametrize("sides,L,B,H,D,seed", [
    (SIDES_TINY, 1, 1, 4, 64, 0), (SIDES_TINY, 2, 2, 3, 64, 1), (SIDES_1024, 2, 2, 3, 128, 2),
    (SIDES_1024, 3, 1, 5, 64, 3)])
def test_compaction_bit_exact(sides, L, B, H, D, seed):
    T = synth.n_tokens(sides)
    kbits = synth.normal_bf16_bits(synth.derive_key(50, seed, 1), (L, B, H, T, D))
    vbits = synth.normal_bf16_bits(synth.derive_key(50, seed, 2), (L, B, H, T, D))
    keep = np.random.default_rng(seed).integers(0, 2, size=(L, H, len(sides))).astype(np.uint8)
    keep[:, :, :2] = 1
    tab = Tables(keep, sides, B, D)
    kc, vc = compact(dev_bf16(kbits), dev_bf16(vbits), tab, sides)
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kref, vref = oracle.compact_kv(kbits, vbits, keep, sides, ho, so, lb)
    assert np.array_equal(bits_of(kc)[:tab.total], kref)
    assert np.array_equal(bits_of(vc)[:tab.total], vref)


def test_compaction_identity_coded_and_untouched_tail():
    """Coded source words; the destination must decode to the right rows and
    nothing past layer_base[L] may be written."""
    sides = SIDES_1024
    g = oracle.ScaleGeometry(sides)
    L, B, H, D = 2, 2, 2, 64
    T = g.T
    rows = np.arange(L * B * H * T, dtype=np.int64).reshape(L, B, H, T)
    kbits = np.zeros((L, B, H, T, D), dtype=np.uint16)
    for d in range(D):
        kbits[..., d] = ((rows * 131 + d * 7) & 0xFFFF).astype(np.uint16)
    vbits = (0xFFFF - kbits).astype(np.uint16)
    keep = np.array([[[1, 1, 0, 1, 0, 1, 1, 0, 0, 1, 0, 1, 0], [1, 1, 1, 0, 0, 0, 0, 0, 0, 0, 0, 0, 1]],
                     [[1, 1, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0], [1] * 13]], dtype=np.uint8)
    tab = Tables(keep, sides, B, D)
    kc = torch.full((tab.total + 4096,), -7.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full((tab.total + 4096,), -7.0, dtype=torch.bfloat16, device="cuda")
    import kv_cache_compression_cas_b200 as vark
    vark.vark_compact_kv(dev_bf16(kbits), dev_bf16(vbits), B * H * T * D, L, B, H, sides, D, tab.keep,
                         tab.head_off, tab.seg_off, tab.layer_base, kc, vc)
    kb, vb = bits_of(kc), bits_of(vc)
    ho, so, pl, lb = oracle.build_offsets(keep, sides, B, D)
    kref, vref = oracle.compact_kv(kbits, vbits, keep, sides, ho, so, lb)
    assert np.array_equal(kb[:tab.total], kref) and np.array_equal(vb[:tab.total], vref)
    tail = np.full(4096, bits_of(torch.tensor([-7.0], dtype=torch.bfloat16))[0], dtype=np.uint16)
    assert np.array_equal(kb[tab.total:], tail) and np.array_equal(vb[tab.total:], tail)
