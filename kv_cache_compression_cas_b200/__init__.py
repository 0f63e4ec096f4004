"""Python binding of the vark C ABI (include/vark.h): head-scale KV-cache
pruning for next-scale (VAR) transformers on B200.

Argument marshalling only -- every step of the path runs in the CUDA library
`libvark.so` built in-tree from `csrc/` (see `build.py`).  Functions carry the
C names; torch tensors supply device memory, `torch.cuda.current_stream()`
the stream.  A missing library raises at first use; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvark.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "vark.h")

VARK_OK = 0
STATUS_NAMES = {0: "VARK_OK", -1: "VARK_E_ARG", -2: "VARK_E_SHAPE", -3: "VARK_E_ALIGN", -4: "VARK_E_BUDGET",
                -5: "VARK_E_CUDA", -6: "VARK_E_TIMEOUT", -7: "VARK_E_DEVICE"}

_lib = None


class VarkError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)} "
                         f"({_load().vark_status_string(self.status).decode()})")


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_U32 = ctypes.c_uint32

_SIGNATURES = {
    "vark_status_string": (ctypes.c_char_p, [_I]),
    "vark_version": (_I, []),
    "vark_scas_accumulate": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "vark_scas_finalize": (_I, [_P, _I, _I, _I, _I, _P]),
    "vark_build_schedule": (_I, [_P, _I, _I, _I, _P, _U32, _I, _P]),
    "vark_build_offsets": (_I, [_P, _I, _I, _I, _P, _I, _I, _P, _P, _P, _P, _P]),
    "vark_compact_kv": (_I, [_P, _P, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "vark_pruned_attention": (_I, [_P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P,
                                   _P, _P]),
    "vark_pruned_attention_step": (_I, [_P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P,
                                        _P, _P, _P]),
    "vark_append_scale": (_I, [_P, _P, _I64, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P]),
    "vark_cache_size_after_layer": (_I, [_P, _I, _I, _I, _P, _I, _I, _P]),
    "vark_rank_stability": (_I, [_P, _P, _I, _I, _I, _P, _U32, _I, _P, _P]),
    "vark_build_early_pruning_schedule": (_I, [_P, _I, _I, _I, _P, _U32, _I, _P, _P]),
    "vark_recompact_kv": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P]),
    "vark_quantize_kv_int8": (_I, [_P, _P, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "vark_dequantize_layer_int8": (_I, [_P, _P, _P, _P, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "vark_quantize_kv_int4": (_I, [_P, _P, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "vark_dequantize_layer_int4": (_I, [_P, _P, _P, _P, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "vark_quantize_kv_int3": (_I, [_P, _P, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "vark_dequantize_layer_int3": (_I, [_P, _P, _P, _P, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "vark_pruned_attention_int8": (_I, [_P, _P, _P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P,
                                        _P, _P, _P, _P]),
    "vark_pruned_attention_int4": (_I, [_P, _P, _P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P,
                                        _P, _P, _P, _P]),
    "vark_pruned_attention_int3": (_I, [_P, _P, _P, _P, _P, _I64, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P,
                                        _P, _P, _P, _P]),
}


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m kv_cache_compression_cas_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def library():
    """The loaded ctypes library."""
    return _load()


def header_symbols():
    """Names of the functions declared in include/vark.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(vark_\w+)\s*\(", text, re.M)))


def _check(rc: int, where: str):
    if rc != VARK_OK:
        raise VarkError(rc, where)


def _sides_arg(sides):
    arr = np.ascontiguousarray(np.asarray(sides, dtype=np.int32))
    return arr, arr.ctypes.data


def _dptr(t, dtype=None, name="tensor"):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _need(t, name, shape=None, numel=None, at_least=None):
    """Size check of a tensor argument against the shape the C call is given,
    made before any pointer is taken: a mismatch would otherwise send the
    kernels' tensor maps, atomics or stores outside the allocation."""
    if t is None:
        return
    got = tuple(t.shape)
    if shape is not None and got != tuple(int(x) for x in shape):
        raise ValueError(f"{name}: shape {got}, expected {tuple(int(x) for x in shape)}")
    if numel is not None and t.numel() != int(numel):
        raise ValueError(f"{name}: {t.numel()} elements, expected {int(numel)}")
    if at_least is not None and t.numel() < int(at_least):
        raise ValueError(f"{name}: {t.numel()} elements, at least {int(at_least)} needed")


def _tokens(sides):
    return int(sum(int(x) * int(x) for x in sides))


def _dims(t, n, name):
    if t is None or len(t.shape) != n:
        raise ValueError(f"{name} must have {n} dimensions")
    return tuple(int(x) for x in t.shape)


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ------------------------------------------------------------------ C ABI calls
def vark_status_string(status: int) -> str:
    return _load().vark_status_string(int(status)).decode()


def vark_version() -> int:
    return int(_load().vark_version())


def vark_scas_accumulate(q, k, v, sides, tau, bias, mass, out=None, dev_status=None, stream=None):
    """S-CAS calibration attention of one layer (see vark.h).  q/k/v bf16
    [B][H][T][D]; tau fp32 [H]; bias fp32 [H][S] or None; mass fp32 [H][S][S]
    accumulated; out bf16 like q or None; dev_status int32 [1]."""
    import torch
    B, H, T, D = _dims(q, 4, "q")
    S = len(sides)
    if T != _tokens(sides):
        raise ValueError(f"q: {T} rows per (batch, head), the scale list has {_tokens(sides)} tokens")
    for t, nm in ((k, "k"), (v, "v"), (out, "out")):
        _need(t, nm, shape=(B, H, T, D))
    _need(tau, "tau", numel=H)
    _need(bias, "bias", numel=H * S)
    _need(mass, "mass", numel=H * S * S)
    _need(dev_status, "dev_status", at_least=1)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_scas_accumulate(
        _dptr(q, torch.bfloat16, "q"), _dptr(k, torch.bfloat16, "k"), _dptr(v, torch.bfloat16, "v"),
        B, H, D, len(s_arr), s_ptr, _dptr(tau, torch.float32, "tau"), _dptr(bias, torch.float32, "bias"),
        _dptr(mass, torch.float32, "mass"), _dptr(out, torch.bfloat16, "out"),
        _dptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(rc, "vark_scas_accumulate")


def vark_scas_finalize(mass: np.ndarray, n_calls: int = 1) -> np.ndarray:
    """Host: S-CAS [L][H][S] fp64 from accumulated mass [L][H][S][S] fp32."""
    m = np.ascontiguousarray(mass, dtype=np.float32)
    if m.ndim == 3:
        m = m[None]
    L, H, S, _ = m.shape
    out = np.zeros((L, H, S), dtype=np.float64)
    _check(_load().vark_scas_finalize(m.ctypes.data, L, H, S, int(n_calls), out.ctypes.data), "vark_scas_finalize")
    return out


def vark_build_schedule(scas: np.ndarray, sides, budget_bp: int, n_sinks: int) -> np.ndarray:
    """Host: keep uint8 [L][H][S] for a budget in basis points."""
    sc = np.ascontiguousarray(scas, dtype=np.float64)
    L, H, S = sc.shape
    s_arr, s_ptr = _sides_arg(sides)
    keep = np.zeros((L, H, S), dtype=np.uint8)
    _check(_load().vark_build_schedule(sc.ctypes.data, L, H, S, s_ptr, int(budget_bp), int(n_sinks),
                                       keep.ctypes.data), "vark_build_schedule")
    return keep


def vark_build_offsets(keep, sides, B: int, D: int, head_off, seg_off, past_len, layer_base, stream=None):
    """Device: offset tables into caller-provided int32/int64 tensors."""
    import torch
    L, H, S = _dims(keep, 3, "keep")
    if S != len(sides):
        raise ValueError(f"keep has {S} scales, the scale list {len(sides)}")
    _need(head_off, "head_off", numel=L * H)
    _need(seg_off, "seg_off", numel=L * H * S)
    _need(past_len, "past_len", numel=L * H * S)
    _need(layer_base, "layer_base", numel=L + 1)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_build_offsets(
        _dptr(keep, torch.uint8, "keep"), L, H, S, s_ptr, int(B), int(D),
        _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
        _dptr(past_len, torch.int32, "past_len"), _dptr(layer_base, torch.int64, "layer_base"), _stream(stream))
    _check(rc, "vark_build_offsets")


def _layer_tables(keep, head_off, seg_off, layer_base, L, H, sides):
    S = len(sides)
    _need(keep, "keep", numel=L * H * S)
    _need(head_off, "head_off", numel=L * H)
    _need(seg_off, "seg_off", numel=L * H * S)
    _need(layer_base, "layer_base", numel=L + 1)


def _dense_source(k, v, layer_stride, L, per_layer):
    if int(layer_stride) < per_layer:
        raise ValueError(f"layer_stride {layer_stride} < {per_layer} elements of one layer")
    need = (int(L) - 1) * int(layer_stride) + per_layer
    _need(k, "k", at_least=need)
    _need(v, "v", at_least=need)


def vark_compact_kv(k, v, layer_stride: int, L: int, B: int, H: int, sides, D: int, keep, head_off, seg_off,
                    layer_base, kc, vc, stream=None):
    """Device: gather retained scale blocks of all layers into kc / vc (each
    must hold layer_base[L] elements)."""
    import torch
    _layer_tables(keep, head_off, seg_off, layer_base, L, H, sides)
    _dense_source(k, v, layer_stride, L, B * H * _tokens(sides) * D)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_compact_kv(
        _dptr(k, torch.bfloat16, "k"), _dptr(v, torch.bfloat16, "v"), int(layer_stride), int(L), int(B), int(H),
        len(s_arr), int(D), s_ptr, _dptr(keep, torch.uint8, "keep"), _dptr(head_off, torch.int32, "head_off"),
        _dptr(seg_off, torch.int32, "seg_off"), _dptr(layer_base, torch.int64, "layer_base"),
        _dptr(kc, torch.bfloat16, "kc"), _dptr(vc, torch.bfloat16, "vc"), _stream(stream))
    _check(rc, "vark_compact_kv")


def _pruned_common_sizes(q, out, kc, vc, kc_rows, head_off, seg_off, past_len, tau, bias, dev_status, qshape,
                         H, S):
    _need(q, "q", shape=qshape)
    _need(out, "out", shape=qshape)
    if int(kc_rows) < 0 or int(kc_rows) % qshape[0] != 0:
        raise ValueError(f"kc_rows {kc_rows} must be a non-negative multiple of the batch")
    if int(kc_rows) > 0:
        if kc is None or vc is None:
            raise ValueError("kc and vc are required when kc_rows > 0")
        _need(kc, "kc", at_least=int(kc_rows) * qshape[3])
        _need(vc, "vc", at_least=int(kc_rows) * qshape[3])
    _need(head_off, "head_off", numel=H)
    _need(seg_off, "seg_off", numel=H * S)
    _need(past_len, "past_len", numel=H * S)
    _need(tau, "tau", numel=H)
    _need(bias, "bias", numel=H * S)
    _need(dev_status, "dev_status", at_least=1)


def vark_pruned_attention(q, kc, vc, kc_rows: int, k_dense, v_dense, sides, query_scale: int, head_off, seg_off,
                          past_len, tau, bias, out, dev_status, stream=None):
    """Device: pruned-cache attention of one layer (see vark.h)."""
    import torch
    B, H, T, D = _dims(k_dense, 4, "k_dense")
    if T != _tokens(sides):
        raise ValueError(f"k_dense: {T} rows per (batch, head), the scale list has {_tokens(sides)} tokens")
    if not -1 <= int(query_scale) < len(sides):
        raise ValueError(f"query_scale {query_scale} out of range")
    Tq = T if int(query_scale) < 0 else int(sides[query_scale]) ** 2
    _need(v_dense, "v_dense", shape=(B, H, T, D))
    _pruned_common_sizes(q, out, kc, vc, kc_rows, head_off, seg_off, past_len, tau, bias, dev_status,
                         (B, H, Tq, D), H, len(sides))
    s_arr, s_ptr = _sides_arg(sides)
    kcp = kc.data_ptr() if (kc is not None and kc_rows > 0) else None
    vcp = vc.data_ptr() if (vc is not None and kc_rows > 0) else None
    if kc is not None:
        _dptr(kc, torch.bfloat16, "kc")
        _dptr(vc, torch.bfloat16, "vc")
    rc = _load().vark_pruned_attention(
        _dptr(q, torch.bfloat16, "q"), kcp, vcp, int(kc_rows),
        _dptr(k_dense, torch.bfloat16, "k_dense"), _dptr(v_dense, torch.bfloat16, "v_dense"),
        int(B), int(H), len(s_arr), int(D), s_ptr, int(query_scale),
        _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
        _dptr(past_len, torch.int32, "past_len"), _dptr(tau, torch.float32, "tau"),
        _dptr(bias, torch.float32, "bias"), _dptr(out, torch.bfloat16, "out"),
        _dptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(rc, "vark_pruned_attention")


def vark_append_scale(k_new, v_new, layer_stride: int, L: int, B: int, H: int, sides, D: int, scale: int, keep,
                      head_off, seg_off, layer_base, kc, vc, stream=None):
    """Device: append scale `scale` of every layer to the compacted cache."""
    import torch
    if not 0 <= int(scale) < len(sides):
        raise ValueError(f"scale {scale} out of range")
    _layer_tables(keep, head_off, seg_off, layer_base, L, H, sides)
    _dense_source(k_new, v_new, layer_stride, L, B * H * int(sides[scale]) ** 2 * D)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_append_scale(
        _dptr(k_new, torch.bfloat16, "k_new"), _dptr(v_new, torch.bfloat16, "v_new"), int(layer_stride), int(L),
        int(B), int(H), len(s_arr), int(D), s_ptr, int(scale), _dptr(keep, torch.uint8, "keep"),
        _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
        _dptr(layer_base, torch.int64, "layer_base"), _dptr(kc, torch.bfloat16, "kc"),
        _dptr(vc, torch.bfloat16, "vc"), _stream(stream))
    _check(rc, "vark_append_scale")


def vark_pruned_attention_step(q, kc, vc, kc_rows: int, k_local, v_local, sides, scale: int, head_off, seg_off,
                               past_len, tau, bias, out, dev_status, stream=None):
    """Device: pruned attention for the queries of the scale being generated."""
    import torch
    B, H, nk, D = _dims(k_local, 4, "k_local")
    if not 0 <= int(scale) < len(sides) or nk != int(sides[scale]) ** 2:
        raise ValueError(f"k_local holds {nk} rows per (batch, head), scale {scale} has a different size")
    _need(v_local, "v_local", shape=(B, H, nk, D))
    _pruned_common_sizes(q, out, kc, vc, kc_rows, head_off, seg_off, past_len, tau, bias, dev_status,
                         (B, H, nk, D), H, len(sides))
    s_arr, s_ptr = _sides_arg(sides)
    kcp = kc.data_ptr() if (kc is not None and kc_rows > 0) else None
    vcp = vc.data_ptr() if (vc is not None and kc_rows > 0) else None
    if kc is not None:
        _dptr(kc, torch.bfloat16, "kc")
        _dptr(vc, torch.bfloat16, "vc")
    rc = _load().vark_pruned_attention_step(
        _dptr(q, torch.bfloat16, "q"), kcp, vcp, int(kc_rows),
        _dptr(k_local, torch.bfloat16, "k_local"), _dptr(v_local, torch.bfloat16, "v_local"),
        int(B), int(H), len(s_arr), int(D), s_ptr, int(scale),
        _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
        _dptr(past_len, torch.int32, "past_len"), _dptr(tau, torch.float32, "tau"),
        _dptr(bias, torch.float32, "bias"), _dptr(out, torch.bfloat16, "out"),
        _dptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(rc, "vark_pruned_attention_step")


def vark_cache_size_after_layer(keep: np.ndarray, sides, B: int, D: int) -> np.ndarray:
    """Host: int64 [S][L] retained K+V bytes after layer l during scale k."""
    kp = np.ascontiguousarray(keep, dtype=np.uint8)
    L, H, S = kp.shape
    s_arr, s_ptr = _sides_arg(sides)
    out = np.zeros((S, L), dtype=np.int64)
    _check(_load().vark_cache_size_after_layer(kp.ctypes.data, L, H, S, s_ptr, int(B), int(D), out.ctypes.data),
           "vark_cache_size_after_layer")
    return out


def vark_rank_stability(scas_a: np.ndarray, scas_b: np.ndarray, sides, budget_bp: int, n_sinks: int):
    """Host: (spearman, drop_jaccard) of two S-CAS arrays [L][H][S]."""
    a = np.ascontiguousarray(scas_a, dtype=np.float64)
    b = np.ascontiguousarray(scas_b, dtype=np.float64)
    L, H, S = a.shape
    s_arr, s_ptr = _sides_arg(sides)
    sp = ctypes.c_double()
    jc = ctypes.c_double()
    _check(_load().vark_rank_stability(a.ctypes.data, b.ctypes.data, L, H, S, s_ptr, int(budget_bp), int(n_sinks),
                                       ctypes.byref(sp), ctypes.byref(jc)), "vark_rank_stability")
    return sp.value, jc.value


def vark_build_early_pruning_schedule(scas: np.ndarray, sides, budget_bp: int, n_sinks: int):
    """Host: (prefix_len int32 [S], evict_step uint8 [L][H][S])."""
    sc = np.ascontiguousarray(scas, dtype=np.float64)
    L, H, S = sc.shape
    s_arr, s_ptr = _sides_arg(sides)
    prefix = np.zeros(S, dtype=np.int32)
    evict = np.zeros((L, H, S), dtype=np.uint8)
    _check(_load().vark_build_early_pruning_schedule(sc.ctypes.data, L, H, S, s_ptr, int(budget_bp), int(n_sinks),
                                                     prefix.ctypes.data, evict.ctypes.data),
           "vark_build_early_pruning_schedule")
    return prefix, evict


def vark_recompact_kv(kc_old, vc_old, head_off_old, seg_off_old, layer_base_old, L: int, B: int, H: int, sides,
                      D: int, max_scale: int, keep_new, head_off_new, seg_off_new, layer_base_new, kc_new, vc_new,
                      stream=None):
    """Device: move a compacted cache into the layout of a new retained set
    (kc_new / vc_new must hold layer_base_new[L] elements)."""
    import torch
    S = len(sides)
    _need(head_off_old, "head_off_old", numel=L * H)
    _need(seg_off_old, "seg_off_old", numel=L * H * S)
    _need(layer_base_old, "layer_base_old", numel=L + 1)
    _layer_tables(keep_new, head_off_new, seg_off_new, layer_base_new, L, H, sides)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_recompact_kv(
        _dptr(kc_old, torch.bfloat16, "kc_old"), _dptr(vc_old, torch.bfloat16, "vc_old"),
        _dptr(head_off_old, torch.int32, "head_off_old"), _dptr(seg_off_old, torch.int32, "seg_off_old"),
        _dptr(layer_base_old, torch.int64, "layer_base_old"), int(L), int(B), int(H), len(s_arr), int(D), s_ptr,
        int(max_scale), _dptr(keep_new, torch.uint8, "keep_new"), _dptr(head_off_new, torch.int32, "head_off_new"),
        _dptr(seg_off_new, torch.int32, "seg_off_new"), _dptr(layer_base_new, torch.int64, "layer_base_new"),
        _dptr(kc_new, torch.bfloat16, "kc_new"), _dptr(vc_new, torch.bfloat16, "vc_new"), _stream(stream))
    _check(rc, "vark_recompact_kv")


def vark_quantize_kv_int8(k, v, layer_stride: int, L: int, B: int, H: int, sides, D: int, keep, head_off, seg_off,
                          layer_base, kq, vq, k_absmax, v_absmax, stream=None):
    """Device: compaction into int8 codes + per-(block, channel) absmax (kq /
    vq must hold layer_base[L] bytes)."""
    import torch
    _layer_tables(keep, head_off, seg_off, layer_base, L, H, sides)
    _dense_source(k, v, layer_stride, L, B * H * _tokens(sides) * D)
    _need(k_absmax, "k_absmax", numel=L * B * H * len(sides) * D)
    _need(v_absmax, "v_absmax", numel=L * B * H * len(sides) * D)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_quantize_kv_int8(
        _dptr(k, torch.bfloat16, "k"), _dptr(v, torch.bfloat16, "v"), int(layer_stride), int(L), int(B), int(H),
        len(s_arr), int(D), s_ptr, _dptr(keep, torch.uint8, "keep"), _dptr(head_off, torch.int32, "head_off"),
        _dptr(seg_off, torch.int32, "seg_off"), _dptr(layer_base, torch.int64, "layer_base"),
        _dptr(kq, torch.int8, "kq"), _dptr(vq, torch.int8, "vq"), _dptr(k_absmax, torch.float32, "k_absmax"),
        _dptr(v_absmax, torch.float32, "v_absmax"), _stream(stream))
    _check(rc, "vark_quantize_kv_int8")


def vark_dequantize_layer_int8(kq, vq, k_absmax, v_absmax, kc_rows: int, B: int, H: int, sides, D: int, head_off,
                               seg_off, kc, vc, stream=None):
    """Device: one layer's int8 codes back to its bf16 compacted block."""
    import torch
    S = len(sides)
    for t, nm in ((kq, "kq"), (vq, "vq"), (kc, "kc"), (vc, "vc")):
        _need(t, nm, at_least=int(kc_rows) * D)
    _need(k_absmax, "k_absmax", numel=B * H * S * D)
    _need(v_absmax, "v_absmax", numel=B * H * S * D)
    _need(head_off, "head_off", numel=H)
    _need(seg_off, "seg_off", numel=H * S)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_dequantize_layer_int8(
        _dptr(kq, torch.int8, "kq"), _dptr(vq, torch.int8, "vq"), _dptr(k_absmax, torch.float32, "k_absmax"),
        _dptr(v_absmax, torch.float32, "v_absmax"), int(kc_rows), int(B), int(H), len(s_arr), int(D), s_ptr,
        _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
        _dptr(kc, torch.bfloat16, "kc"), _dptr(vc, torch.bfloat16, "vc"), _stream(stream))
    _check(rc, "vark_dequantize_layer_int8")


def vark_quantize_kv_int4(k, v, layer_stride: int, L: int, B: int, H: int, sides, D: int, keep, head_off, seg_off,
                          layer_base, kq, vq, k_scale, v_scale, stream=None):
    """Device: compaction into packed 4-bit codes + per-(block, channel) bf16
    scales (kq / vq must hold layer_base[L] / 2 bytes)."""
    import torch
    _layer_tables(keep, head_off, seg_off, layer_base, L, H, sides)
    _dense_source(k, v, layer_stride, L, B * H * _tokens(sides) * D)
    _need(k_scale, "k_scale", numel=L * B * H * len(sides) * D)
    _need(v_scale, "v_scale", numel=L * B * H * len(sides) * D)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_quantize_kv_int4(
        _dptr(k, torch.bfloat16, "k"), _dptr(v, torch.bfloat16, "v"), int(layer_stride), int(L), int(B), int(H),
        len(s_arr), int(D), s_ptr, _dptr(keep, torch.uint8, "keep"), _dptr(head_off, torch.int32, "head_off"),
        _dptr(seg_off, torch.int32, "seg_off"), _dptr(layer_base, torch.int64, "layer_base"),
        _dptr(kq, torch.uint8, "kq"), _dptr(vq, torch.uint8, "vq"), _dptr(k_scale, torch.int16, "k_scale"),
        _dptr(v_scale, torch.int16, "v_scale"), _stream(stream))
    _check(rc, "vark_quantize_kv_int4")


def vark_dequantize_layer_int4(kq, vq, k_scale, v_scale, kc_rows: int, B: int, H: int, sides, D: int, head_off,
                               seg_off, kc, vc, stream=None):
    """Device: one layer's packed 4-bit codes back to its bf16 compacted block."""
    import torch
    S = len(sides)
    _need(kq, "kq", at_least=int(kc_rows) * D // 2)
    _need(vq, "vq", at_least=int(kc_rows) * D // 2)
    for t, nm in ((kc, "kc"), (vc, "vc")):
        _need(t, nm, at_least=int(kc_rows) * D)
    _need(k_scale, "k_scale", numel=B * H * S * D)
    _need(v_scale, "v_scale", numel=B * H * S * D)
    _need(head_off, "head_off", numel=H)
    _need(seg_off, "seg_off", numel=H * S)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_dequantize_layer_int4(
        _dptr(kq, torch.uint8, "kq"), _dptr(vq, torch.uint8, "vq"), _dptr(k_scale, torch.int16, "k_scale"),
        _dptr(v_scale, torch.int16, "v_scale"), int(kc_rows), int(B), int(H), len(s_arr), int(D), s_ptr,
        _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
        _dptr(kc, torch.bfloat16, "kc"), _dptr(vc, torch.bfloat16, "vc"), _stream(stream))
    _check(rc, "vark_dequantize_layer_int4")


def vark_quantize_kv_int3(k, v, layer_stride: int, L: int, B: int, H: int, sides, D: int, keep, head_off, seg_off,
                          layer_base, kq, vq, k_scale, v_scale, stream=None):
    """Device: compaction into 3-bit codes (24-bit groups of 8 channels) +
    per-(block, channel) bf16 scales (kq / vq must hold 3 layer_base[L] / 8 bytes)."""
    import torch
    _layer_tables(keep, head_off, seg_off, layer_base, L, H, sides)
    _dense_source(k, v, layer_stride, L, B * H * _tokens(sides) * D)
    _need(k_scale, "k_scale", numel=L * B * H * len(sides) * D)
    _need(v_scale, "v_scale", numel=L * B * H * len(sides) * D)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_quantize_kv_int3(
        _dptr(k, torch.bfloat16, "k"), _dptr(v, torch.bfloat16, "v"), int(layer_stride), int(L), int(B), int(H),
        len(s_arr), int(D), s_ptr, _dptr(keep, torch.uint8, "keep"), _dptr(head_off, torch.int32, "head_off"),
        _dptr(seg_off, torch.int32, "seg_off"), _dptr(layer_base, torch.int64, "layer_base"),
        _dptr(kq, torch.uint8, "kq"), _dptr(vq, torch.uint8, "vq"), _dptr(k_scale, torch.int16, "k_scale"),
        _dptr(v_scale, torch.int16, "v_scale"), _stream(stream))
    _check(rc, "vark_quantize_kv_int3")


def vark_dequantize_layer_int3(kq, vq, k_scale, v_scale, kc_rows: int, B: int, H: int, sides, D: int, head_off,
                               seg_off, kc, vc, stream=None):
    """Device: one layer's 3-bit codes back to its bf16 compacted block."""
    import torch
    S = len(sides)
    _need(kq, "kq", at_least=int(kc_rows) * 3 * D // 8)
    _need(vq, "vq", at_least=int(kc_rows) * 3 * D // 8)
    for t, nm in ((kc, "kc"), (vc, "vc")):
        _need(t, nm, at_least=int(kc_rows) * D)
    _need(k_scale, "k_scale", numel=B * H * S * D)
    _need(v_scale, "v_scale", numel=B * H * S * D)
    _need(head_off, "head_off", numel=H)
    _need(seg_off, "seg_off", numel=H * S)
    s_arr, s_ptr = _sides_arg(sides)
    rc = _load().vark_dequantize_layer_int3(
        _dptr(kq, torch.uint8, "kq"), _dptr(vq, torch.uint8, "vq"), _dptr(k_scale, torch.int16, "k_scale"),
        _dptr(v_scale, torch.int16, "v_scale"), int(kc_rows), int(B), int(H), len(s_arr), int(D), s_ptr,
        _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
        _dptr(kc, torch.bfloat16, "kc"), _dptr(vc, torch.bfloat16, "vc"), _stream(stream))
    _check(rc, "vark_dequantize_layer_int3")


def _pruned_packed(bits, q, kq, vq, k_tab, v_tab, kc_rows: int, k_dense, v_dense, sides, query_scale: int,
                   head_off, seg_off, past_len, tau, bias, out, dev_status, stream):
    import torch
    B, H, T, D = _dims(k_dense, 4, "k_dense")
    S = len(sides)
    if T != _tokens(sides):
        raise ValueError(f"k_dense: {T} rows per (batch, head), the scale list has {_tokens(sides)} tokens")
    if not -1 <= int(query_scale) < S:
        raise ValueError(f"query_scale {query_scale} out of range")
    Tq = T if int(query_scale) < 0 else int(sides[query_scale]) ** 2
    _need(v_dense, "v_dense", shape=(B, H, T, D))
    _pruned_common_sizes(q, out, None, None, 0, head_off, seg_off, past_len, tau, bias, dev_status,
                         (B, H, Tq, D), H, S)
    if int(kc_rows) < 0 or int(kc_rows) % B != 0:
        raise ValueError(f"kc_rows {kc_rows} must be a non-negative multiple of the batch")
    code_t, tab_t = (torch.int8, torch.float32) if bits == 8 else (torch.uint8, torch.int16)
    _need(kq, "kq", at_least=int(kc_rows) * bits * D // 8)
    _need(vq, "vq", at_least=int(kc_rows) * bits * D // 8)
    _need(k_tab, "k_tab", numel=B * H * S * D)
    _need(v_tab, "v_tab", numel=B * H * S * D)
    s_arr, s_ptr = _sides_arg(sides)
    fn = getattr(_load(), f"vark_pruned_attention_int{bits}")
    rc = fn(_dptr(q, torch.bfloat16, "q"), _dptr(kq, code_t, "kq"), _dptr(vq, code_t, "vq"),
            _dptr(k_tab, tab_t, "k_tab"), _dptr(v_tab, tab_t, "v_tab"), int(kc_rows),
            _dptr(k_dense, torch.bfloat16, "k_dense"), _dptr(v_dense, torch.bfloat16, "v_dense"),
            int(B), int(H), len(s_arr), int(D), s_ptr, int(query_scale),
            _dptr(head_off, torch.int32, "head_off"), _dptr(seg_off, torch.int32, "seg_off"),
            _dptr(past_len, torch.int32, "past_len"), _dptr(tau, torch.float32, "tau"),
            _dptr(bias, torch.float32, "bias"), _dptr(out, torch.bfloat16, "out"),
            _dptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(rc, f"vark_pruned_attention_int{bits}")


def vark_pruned_attention_int8(q, kq, vq, k_absmax, v_absmax, kc_rows: int, k_dense, v_dense, sides,
                               query_scale: int, head_off, seg_off, past_len, tau, bias, out, dev_status,
                               stream=None):
    """Device: pruned attention of one layer straight over its 8-bit codes
    (kq / vq at the layer's first code, k_absmax / v_absmax the layer's
    [B][H][S][D] tables); the past is dequantised inside the kernel."""
    _pruned_packed(8, q, kq, vq, k_absmax, v_absmax, kc_rows, k_dense, v_dense, sides, query_scale, head_off,
                   seg_off, past_len, tau, bias, out, dev_status, stream)


def vark_pruned_attention_int4(q, kq, vq, k_scale, v_scale, kc_rows: int, k_dense, v_dense, sides,
                               query_scale: int, head_off, seg_off, past_len, tau, bias, out, dev_status,
                               stream=None):
    """Device: pruned attention of one layer straight over its packed 4-bit codes."""
    _pruned_packed(4, q, kq, vq, k_scale, v_scale, kc_rows, k_dense, v_dense, sides, query_scale, head_off,
                   seg_off, past_len, tau, bias, out, dev_status, stream)


def vark_pruned_attention_int3(q, kq, vq, k_scale, v_scale, kc_rows: int, k_dense, v_dense, sides,
                               query_scale: int, head_off, seg_off, past_len, tau, bias, out, dev_status,
                               stream=None):
    """Device: pruned attention of one layer straight over its 3-bit codes (D = 128)."""
    _pruned_packed(3, q, kq, vq, k_scale, v_scale, kc_rows, k_dense, v_dense, sides, query_scale, head_off,
                   seg_off, past_len, tau, bias, out, dev_status, stream)
