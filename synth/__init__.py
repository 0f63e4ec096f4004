"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module holds no arithmetic of the pruning method.  It only defines the
workloads (scale lists, shapes, budgets) and draws their random inputs:

* bf16 Q/K/V tensors from a counter-based generator that gives identical bits
  on the CPU (NumPy) and on a CUDA device (plain torch integer ops), so a
  full-size tensor can be made on the device while the oracle regenerates any
  sampled subset of it on the host;
* the per-head temperature tau ~ U[0.5, 2] and the additive per-(head, source
  scale) logit bias (1-3 biased scales per head, values U[0, 2]);
* random retained-scale sets for the final-scale sweep.

Generator definition (fixed, so both sides can implement it independently):

    fmix32(x)   = MurmurHash3's 32-bit finaliser (x ^= x>>16; x *= 0x85EBCA6B;
                  x ^= x>>13; x *= 0xC2B2AE35; x ^= x>>16), arithmetic mod 2^32
    word(key, i, j) = fmix32(lo(i) ^ fmix32((hi(i) * 0x9E3779B9 + kj) mod 2^32))
                  with kj = fmix32(key ^ fmix32(j + 1)), lo/hi the 32-bit halves
                  of the flat C-order element index i, j = 0..5
    z(i)        = (sum over j of the two 16-bit halves of word(key, i, j) + 6)
                  * 2^-16 - 6                     (Irwin-Hall sum of 12 uniforms)
    value(i)    = bf16 round-to-nearest-even of z(i) (exact in fp32)

z has mean 0 and variance 1 and is bounded by +-6: it stands in for the N(0, 1)
inputs of the workloads.  Every step is integer arithmetic or an exact fp32
operation, so the two implementations agree bit for bit.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Sequence

import numpy as np

MASK32 = 0xFFFFFFFF

# Scale side lists.  Token maps are square; scale s holds side_s^2 tokens in
# raster order, and the scales are stored in ascending order.
SIDES_TINY = (1, 2, 3, 4, 5, 6, 8)                                  # 155 tokens
SIDES_1024 = (1, 2, 4, 6, 8, 12, 16, 20, 24, 32, 40, 48, 64)       # 10,521 tokens


# --------------------------------------------------------------------------
# Workload definitions
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  `batch` is the inference batch; calibration
    folds `n_seeds` seeds into the batch of the calibration call."""
    name: str
    sides: tuple
    heads: int
    head_dim: int
    layers: int
    batch: int
    n_seeds: int
    budget_bp: int            # memory budget in basis points of the full cache
    n_sinks: int = 2          # scales 0..n_sinks-1 are never dropped
    with_bias: bool = False   # per-head additive logit bias toward 1-3 scales
    query_scale: int = -1     # -1: every scale's queries; else one scale
    base_seed: int = 0
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload("tiny", SIDES_TINY, heads=4, head_dim=64, layers=1, batch=1,
                     n_seeds=4, budget_bp=5000, base_seed=0),
    "calib_1024": Workload("calib_1024", SIDES_1024, heads=16, head_dim=128, layers=1,
                           batch=1, n_seeds=16, budget_bp=10000, with_bias=True,
                           base_seed=2),
    "pruned_32l": Workload("pruned_32l", SIDES_1024, heads=16, head_dim=128, layers=32,
                           batch=8, n_seeds=16, budget_bp=1000, with_bias=True,
                           base_seed=3),
    "large_8l": Workload("large_8l", SIDES_1024, heads=32, head_dim=128, layers=8,
                         batch=4, n_seeds=8, budget_bp=400, with_bias=True,
                         base_seed=4),
    "final_scale": Workload("final_scale", SIDES_1024, heads=16, head_dim=128, layers=1,
                            batch=1, n_seeds=0, budget_bp=10000, query_scale=12,
                            base_seed=5,
                            extra={"budgets_bp": (10000, 2000, 1000, 400),
                                   "batches": (1, 4, 16, 32)}),
}


def n_tokens(sides: Sequence[int]) -> int:
    return int(sum(int(s) * int(s) for s in sides))


# --------------------------------------------------------------------------
# Counter-based generator, NumPy side
# --------------------------------------------------------------------------
def _mul32(x, c: int):
    """Low 32 bits of x*c for 0 <= x < 2^32 without leaving 49-bit range."""
    c_lo, c_hi = c & 0xFFFF, (c >> 16) & 0xFFFF
    return (x * c_lo + (((x * c_hi) & 0xFFFF) << 16)) & MASK32


def fmix32(x):
    """MurmurHash3 32-bit finaliser on uint64 arrays / Python ints (< 2^32)."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x85EBCA6B)
    x = x ^ (x >> 13)
    x = _mul32(x, 0xC2B2AE35)
    x = x ^ (x >> 16)
    return x


def derive_key(*parts: int) -> int:
    """Fold small non-negative integers into one 32-bit stream key."""
    k = 0x243F6A88
    for p in parts:
        k = fmix32((k ^ (int(p) & MASK32)) & MASK32)
        k = (k + 0x9E3779B9) & MASK32
    return int(k)


def _subkeys(key: int):
    return [int(fmix32((key ^ int(fmix32(j + 1))) & MASK32)) for j in range(6)]


def _normal_f32_from_index_np(key: int, idx: np.ndarray) -> np.ndarray:
    idx = idx.astype(np.uint64)
    lo = idx & np.uint64(MASK32)
    hi = idx >> np.uint64(32)
    acc = np.zeros(idx.shape, dtype=np.uint64)
    for kj in _subkeys(key):
        t = fmix32((_mul32(hi, 0x9E3779B9) + np.uint64(kj)) & np.uint64(MASK32))
        w = fmix32(lo ^ t)
        acc += (w & np.uint64(0xFFFF)) + (w >> np.uint64(16))
    z = (acc + np.uint64(6)).astype(np.float32) * np.float32(2.0 ** -16) - np.float32(6.0)
    return z


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 with round-to-nearest-even; returns uint16 bits.
    (Inputs here are finite.)"""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16_bits(key: int, shape: Sequence[int]) -> np.ndarray:
    """Whole tensor of generator values as uint16 bf16 bits (host)."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    chunk = 1 << 22
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        idx = np.arange(s, e, dtype=np.uint64)
        out[s:e] = f32_to_bf16_bits(_normal_f32_from_index_np(key, idx))
    return out.reshape(tuple(shape))


def normal_bf16_bits_at(key: int, flat_index: np.ndarray) -> np.ndarray:
    """Generator values at selected flat C-order indices (host)."""
    flat_index = np.asarray(flat_index, dtype=np.uint64)
    return f32_to_bf16_bits(_normal_f32_from_index_np(key, flat_index.ravel())).reshape(flat_index.shape)


def rows_bf16_bits(key: int, shape: Sequence[int], lead: Sequence[int], row_lo: int, row_hi: int) -> np.ndarray:
    """Rows [row_lo, row_hi) of the last-but-one axis at leading index `lead`
    of a [..., rows, D] tensor, as uint16 bits [row_hi-row_lo][D]."""
    shape = tuple(int(s) for s in shape)
    D = shape[-1]
    strides = np.cumprod((1,) + shape[::-1][:-1])[::-1]
    base = int(sum(int(i) * int(st) for i, st in zip(lead, strides[: len(lead)])))
    rs = int(strides[-2])
    idx = base + np.arange(row_lo, row_hi, dtype=np.int64)[:, None] * rs + np.arange(D, dtype=np.int64)[None, :]
    return normal_bf16_bits_at(key, idx.astype(np.uint64))


# --------------------------------------------------------------------------
# Counter-based generator, torch side (same definition, any device)
# --------------------------------------------------------------------------
def _t_mul32(x, c: int):
    c_lo, c_hi = c & 0xFFFF, (c >> 16) & 0xFFFF
    return (x * c_lo + (((x * c_hi) & 0xFFFF) << 16)) & MASK32


def _t_fmix32(x):
    x = x ^ (x >> 16)
    x = _t_mul32(x, 0x85EBCA6B)
    x = x ^ (x >> 13)
    x = _t_mul32(x, 0xC2B2AE35)
    x = x ^ (x >> 16)
    return x


def normal_bf16_torch(key: int, shape: Sequence[int], device="cpu", chunk: int = 1 << 26):
    """Whole tensor of generator values as a torch.bfloat16 tensor on `device`.
    Uses only int64 torch ops (values kept below 2^49), so CPU and CUDA agree."""
    import torch
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(n, dtype=torch.int16, device=device)
    subs = _subkeys(key)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        idx = torch.arange(s, e, dtype=torch.int64, device=device)
        lo = idx & MASK32
        hi = idx >> 32
        acc = torch.zeros_like(idx)
        for kj in subs:
            t = _t_fmix32((_t_mul32(hi, 0x9E3779B9) + kj) & MASK32)
            w = _t_fmix32(lo ^ t)
            acc += (w & 0xFFFF) + (w >> 16)
        del lo, hi, idx
        z = (acc + 6).to(torch.float32) * (2.0 ** -16) - 6.0
        b = z.view(torch.int32).to(torch.int64) & MASK32
        r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
        out[s:e] = (r - ((r >> 15) << 16)).to(torch.int16)   # two's complement int16
    return out.view(torch.bfloat16).reshape(shape)


# --------------------------------------------------------------------------
# Small host-side draws (PCG64 via numpy.random.default_rng)
# --------------------------------------------------------------------------
def gen_tau(seed: int, heads: int) -> np.ndarray:
    """Per-head temperature tau_h ~ U[0.5, 2] (fp32)."""
    rng = np.random.default_rng([seed, 0x7A])
    return rng.uniform(0.5, 2.0, size=heads).astype(np.float32)


def gen_bias(seed: int, heads: int, n_scales: int) -> np.ndarray:
    """Per-head additive logit bias toward 1-3 randomly chosen source scales,
    each biased value U[0, 2]; zero elsewhere.  fp32 [heads][n_scales]."""
    rng = np.random.default_rng([seed, 0xB1])
    bias = np.zeros((heads, n_scales), dtype=np.float32)
    for h in range(heads):
        r = int(rng.integers(1, 4))
        chosen = rng.choice(n_scales, size=min(r, n_scales), replace=False)
        bias[h, chosen] = rng.uniform(0.0, 2.0, size=len(chosen)).astype(np.float32)
    return bias


def layer_seed(w: Workload, layer: int) -> int:
    """Seed of the synthetic 'model' parameters (tau, bias) of one layer."""
    return derive_key(w.base_seed, 0x5EED, layer)


def qkv_key(w: Workload, layer: int, which: str, phase: str) -> int:
    """Stream key of a Q/K/V tensor: phase 'calib' (seeds folded into the batch
    axis) or 'infer' (the inference batch)."""
    return derive_key(w.base_seed, {"calib": 1, "infer": 2}[phase], layer, {"q": 1, "k": 2, "v": 3}[which])


def random_scas(seed: int, layers: int, heads: int, n_scales: int) -> np.ndarray:
    """Synthetic S-CAS-shaped scores, fp64 [L][H][S], U[0, 1) with the last
    scale at 0 (no later scale reads it): used where a test needs a schedule at
    full size without running calibration on the host."""
    rng = np.random.default_rng([seed, 0x5C])
    sc = rng.uniform(0.0, 1.0, size=(layers, heads, n_scales))
    sc[:, :, -1] = 0.0
    return sc


def random_keep(seed: int, heads: int, sides: Sequence[int], budget_bp: int,
                n_sinks: int, query_scale: int) -> np.ndarray:
    """Seed-random retained-scale sets for the final-scale sweep, uint8
    [1][heads][S].  Per head: shuffle the past scales n_sinks..query_scale-1,
    walk them and keep a scale while the running token count (sinks
    included) stays within budget_bp/10000 of the full per-head cache; the
    sinks are always kept and the local scale is marked kept (it is always
    attended)."""
    S = len(sides)
    n = [int(s) * int(s) for s in sides]
    full = sum(n)
    keep = np.zeros((1, heads, S), dtype=np.uint8)
    rng = np.random.default_rng([seed, 0xC8])
    for h in range(heads):
        running = sum(n[:n_sinks])
        keep[0, h, :n_sinks] = 1
        order = rng.permutation(np.arange(n_sinks, query_scale))
        for s in order:
            if (running + n[s]) * 10000 <= budget_bp * full:
                keep[0, h, s] = 1
                running += n[s]
        keep[0, h, query_scale] = 1
    return keep
