"""Failure detection on the GPU without a fault: the test hook makes every
CTA's producer withhold one key tile, so the waits on it run out under a
short limit.  The kernels must record VARK_E_TIMEOUT in the status word,
drain their own asynchronous work, free tensor memory and return; the CUDA
context must stay usable (a normal call afterwards matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import kv_cache_compression_cas_b200 as vark
import oracle
import synth
from tests.helpers import Tables, bits_of, compact, dev_bf16, f64, status_word

pytestmark = pytest.mark.gpu

VARK_E_TIMEOUT = -6


def _calib(sides, B, H, D, seed, want_out=True):
    T = synth.n_tokens(sides)
    bits = [synth.normal_bf16_bits(synth.derive_key(90, seed, i), (B, H, T, D)) for i in range(3)]
    tau = synth.gen_tau(seed, H)
    q, k, v = (dev_bf16(b) for b in bits)
    S = len(sides)
    mass = torch.zeros((H, S, S), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q) if want_out else None
    st = status_word()
    vark.vark_scas_accumulate(q, k, v, sides, torch.from_numpy(tau).cuda(), None, mass, out, st)
    torch.cuda.synchronize()
    return int(st.item()), bits, tau, mass, out


def test_withheld_key_tile_times_out_and_context_stays_usable(monkeypatch):
    sides = synth.SIDES_1024
    monkeypatch.setenv("VARK_TEST_WAIT_LIMIT_MS", "100")
    monkeypatch.setenv("VARK_TEST_WITHHOLD_KV_TILE", "3")
    t0 = time.time()
    status, *_ = _calib(sides, 1, 2, 128, 1)
    dt = time.time() - t0
    assert status == VARK_E_TIMEOUT
    assert dt < 30.0
    # S-CAS only (no output: no V, no PV) gives up the same way
    status, *_ = _calib(sides, 1, 2, 128, 1, want_out=False)
    assert status == VARK_E_TIMEOUT
    # pruned attention takes the same path
    B, H, D = 1, 2, 128
    T = synth.n_tokens(sides)
    kb = synth.normal_bf16_bits(synth.derive_key(91, 1), (B, H, T, D))
    keep = np.ones((1, H, len(sides)), dtype=np.uint8)
    tab = Tables(keep, sides, B, D)
    kd = dev_bf16(kb)
    kc, vc = compact(kd[None], kd[None], tab, sides)
    out = torch.empty_like(kd)
    st = status_word()
    vark.vark_pruned_attention(kd, kc, vc, tab.kc_rows(0), kd, kd, sides, -1,
                               tab.head_off[0], tab.seg_off[0], tab.past_len[0],
                               torch.ones(H, dtype=torch.float32, device="cuda"), None, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == VARK_E_TIMEOUT
    # hooks off: the same context computes correct results again
    monkeypatch.delenv("VARK_TEST_WAIT_LIMIT_MS")
    monkeypatch.delenv("VARK_TEST_WITHHOLD_KV_TILE")
    tiny = synth.SIDES_TINY
    status, bits, tau, mass, out = _calib(tiny, 2, 2, 64, 2)
    assert status == 0
    O_ref, m_ref = oracle.block_causal_attention(*(f64(b) for b in bits), tiny, tau.astype(np.float64), None)
    assert np.abs(f64(bits_of(out)) - O_ref).max() <= 2e-2
    np.testing.assert_allclose(mass.cpu().numpy(), oracle.scas_mass(m_ref, tiny), rtol=1e-3)
