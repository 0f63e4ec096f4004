"""Quantised retained cache (int8, per (block, channel) groups).

[VAR-Q] summary page: KV-cache quantisation for visual autoregressive models
with groups indexed by (block, channel), block boundaries given by the
generation loop, composable with cache eviction.  The page's kernels pack
INT2-INT4 codes on A100; this library's reading is the plain 8-bit member of
that grouping: a block is one retained scale of one (layer, batch, head), each
channel d of it has one absmax a, and

    code = rint(x / (a / 127)) clamped to [-127, 127]   (fp32 IEEE division,
           round half to even; a = 0 gives 0)
    x'   = code * (a / 127) in fp32, rounded to bf16.

Parity: exact arithmetic on both sides (bit-exact codes, absmax and
dequantised bf16); pinned by the error bound |x' - x| <= a / 254 (+ bf16
rounding), exactness on a grid of representable values, and zero blocks.
"""
from __future__ import annotations

import numpy as np

from .scales import ScaleGeometry


def _bf16(x32):
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def _f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def quantize_block(x_bits):
    """x_bits: uint16 bf16 [rows][D].  Returns (codes int8 [rows][D], absmax fp32 [D])."""
    x = _f32(x_bits)
    a = np.abs(x).max(axis=0).astype(np.float32)
    sc = (a / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.rint((x / sc[None, :]).astype(np.float32))
    t = np.where(sc[None, :] == 0, 0, t)
    return np.clip(t, -127, 127).astype(np.int8), a


def dequantize_block(codes, absmax):
    sc = (np.asarray(absmax, dtype=np.float32) / np.float32(127.0)).astype(np.float32)
    return _bf16((codes.astype(np.float32) * sc[None, :]).astype(np.float32))


def quantize_kv(k_dense, v_dense, keep, sides, head_off, seg_off, layer_base):
    """Dense uint16 [L][B][H][T][D] -> (kq, vq int8 flat, k_absmax, v_absmax fp32 [L][B][H][S][D])."""
    keep = np.asarray(keep)
    L, B, H, T, D = k_dense.shape
    geom = ScaleGeometry(sides)
    total = int(layer_base[L])
    kq = np.zeros(total, dtype=np.int8)
    vq = np.zeros(total, dtype=np.int8)
    ka = np.zeros((L, B, H, geom.S, D), dtype=np.float32)
    va = np.zeros((L, B, H, geom.S, D), dtype=np.float32)
    for l in range(L):
        R_l = int(layer_base[l + 1] - layer_base[l]) // (B * D)
        for b in range(B):
            for h in range(H):
                for s in range(geom.S):
                    if not keep[l, h, s]:
                        continue
                    sl = slice(geom.off[s], geom.off[s] + geom.n[s])
                    ck, ak = quantize_block(k_dense[l, b, h, sl])
                    cv, av = quantize_block(v_dense[l, b, h, sl])
                    row = b * R_l + int(head_off[l, h]) + int(seg_off[l, h, s])
                    dst = int(layer_base[l]) + row * D
                    kq[dst:dst + geom.n[s] * D] = ck.ravel()
                    vq[dst:dst + geom.n[s] * D] = cv.ravel()
                    ka[l, b, h, s], va[l, b, h, s] = ak, av
    return kq, vq, ka, va
