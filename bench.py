#!/usr/bin/env python3
"""Benchmark of the HeatKV-style pruning hot path on B200.

One step = one pass of the whole path over one batch of synthetic input,
for the pruned-inference workload (32 layers, 16 heads, head_dim 128, 1024^2
scale list, batch 8, 10% budget, sinks 0-1):

  1. S-CAS calibration attention of every layer (16 calibration seeds folded
     into the batch); the attention output O is written, as the layer's
     output in a calibration forward pass        vark_scas_accumulate
  2. S-CAS finalisation and the greedy keep schedule (host) vark_scas_finalize,
                                                           vark_build_schedule
  3. offset tables                                       vark_build_offsets
  4. compaction of all layers' K/V                       vark_compact_kv
  5. pruned-cache attention of every layer, all 13 query scales
                                                         vark_pruned_attention

value = algorithmic attention FLOPs of the step (calibration + pruned) / step
time, inputs resident in HBM.  Per-kernel CUDA-event timings give pruned
attention TFLOP/s and query tokens/s, compaction GB/s and roofline fractions.
e2e repeats the step through the same calls with the inputs copied in from
pinned host memory and the attention outputs copied back each step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vark|reference]

Under torchrun every rank runs an independent replica on its own inputs
(weak scaling); the reported value is the sum of all ranks' work over the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "pruned-cache attention TFLOP/s + query tokens/s; compaction GB/s; % of roofline"
WORKLOAD = "pruned_32l"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "traffic.json")
ATTN_SOURCES = [os.path.join(ROOT, "kv_cache_compression_cas_b200", "csrc", f)
                for f in ("vark_attention.cu", "vark_common.cuh")]


def attention_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in ATTN_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic():
    """(DRAM bytes per full calibration launch, capture note) from the
    committed capture record, or (None, reason) when the attention kernel's
    source has changed since the capture."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)["attn_kernel<128,false,true,true>"]
    except (OSError, KeyError, ValueError):
        return None, "no capture record"
    if rec.get("source_sha16") != attention_source_hash():
        return None, "kernel changed since the capture"
    return int(rec["dram_bytes_per_launch"]), rec.get("capture", "")


# ---------------------------------------------------------------- algorithmic work
def calib_flops(sides, B, H, D):
    n = [s * s for s in sides]
    off = np.cumsum([0] + n[:-1])
    return float(sum(4.0 * n[k] * (off[k] + n[k]) * D for k in range(len(n)))) * B * H


def pruned_flops(keep, sides, B, D):
    """sum over (layer, head, query scale k) of 4 * B * n_k * (kept past rows + n_k) * D."""
    n = np.array([s * s for s in sides], dtype=np.float64)
    L, H, S = keep.shape
    tot = 0.0
    for k in range(S):
        past = (keep[:, :, :k].astype(np.float64) * n[None, None, :k]).sum(axis=2)   # [L][H]
        tot += float((4.0 * B * n[k] * (past + n[k]) * D).sum())
    return tot


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        busy = [x for x in sm if smax and x > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def randn_bf16(shape, seed, device):
    """Seeded N(0, 1) bf16 tensor made on the device, one torch launch per
    leading slice.  (Parity tests use the host-reproducible generator in
    `synth`; the benchmark only needs seeded data of the same distribution.)"""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    t = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for i in range(shape[0]):
        t[i].normal_(generator=g)
    return t


def replica_seed(w: synth.Workload, rank: int) -> int:
    """Seed of one rank's replica: every rank draws its own inputs (weak
    scaling over independent replicas, no data-path exchange)."""
    return synth.derive_key(w.base_seed, 0xBE, rank)


# ---------------------------------------------------------------- the pipeline
class Pipeline:
    """Device buffers and one step of the hot path for one rank."""

    def __init__(self, w: synth.Workload, rank: int, device):
        import torch
        import kv_cache_compression_cas_b200 as vark
        self.vark, self.torch = vark, torch
        self.w, self.dev = w, device
        self.sides = w.sides
        self.S = len(w.sides)
        self.T = synth.n_tokens(w.sides)
        L, B, H, D, T, S = w.layers, w.batch, w.heads, w.head_dim, self.T, self.S
        Bc = w.n_seeds
        seed = replica_seed(w, rank)
        # calibration inputs: per layer [seeds][H][T][D]; inference: [L][B][H][T][D]
        self.cq = randn_bf16((L, Bc, H, T, D), seed + 1, device)
        self.ck = randn_bf16((L, Bc, H, T, D), seed + 2, device)
        self.cv = randn_bf16((L, Bc, H, T, D), seed + 3, device)
        self.q = randn_bf16((L, B, H, T, D), seed + 4, device)
        self.k = randn_bf16((L, B, H, T, D), seed + 5, device)
        self.v = randn_bf16((L, B, H, T, D), seed + 6, device)
        taus = [synth.gen_tau(synth.layer_seed(w, l) + rank, H) for l in range(L)]
        biases = [synth.gen_bias(synth.layer_seed(w, l) + rank, H, S) for l in range(L)]
        self.tau = torch.from_numpy(np.stack(taus)).to(device)
        self.bias = torch.from_numpy(np.stack(biases)).to(device)
        self.mass = torch.zeros((L, H, S, S), dtype=torch.float32, device=device)
        self.cout = torch.empty((Bc, H, T, D), dtype=torch.bfloat16, device=device)   # calibration O, per layer
        self.out = torch.empty_like(self.q)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.keep = torch.empty((L, H, S), dtype=torch.uint8, device=device)
        self.head_off = torch.empty((L, H), dtype=torch.int32, device=device)
        self.seg_off = torch.empty((L, H, S), dtype=torch.int32, device=device)
        self.past_len = torch.empty((L, H, S), dtype=torch.int32, device=device)
        self.layer_base = torch.empty(L + 1, dtype=torch.int64, device=device)
        cap = B * D * (w.budget_bp * L * H * T // 10000 + T)
        self.kc = torch.empty(cap, dtype=torch.bfloat16, device=device)
        self.vc = torch.empty(cap, dtype=torch.bfloat16, device=device)
        self.mass_host = torch.empty((L, H, S, S), dtype=torch.float32, pin_memory=True)
        self.keep_host = torch.empty((L, H, S), dtype=torch.uint8, pin_memory=True)
        self.base_host = torch.empty(L + 1, dtype=torch.int64, pin_memory=True)
        self.calib_flops = calib_flops(self.sides, Bc, H, D) * L
        self.last_keep = None
        self.launches = 0

    def step(self, ev=None):
        """One pass of the hot path.  ev: optional dict of CUDA events to record
        phase boundaries (keys: t0, calib, sched, offs, comp, attn)."""
        torch, vark, w = self.torch, self.vark, self.w
        L, B, H, D, S = w.layers, w.batch, w.heads, w.head_dim, self.S
        st = torch.cuda.current_stream()
        rec = (lambda k: ev[k].record(st)) if ev else (lambda k: None)
        rec("t0")
        self.mass.zero_()
        for l in range(L):
            vark.vark_scas_accumulate(self.cq[l], self.ck[l], self.cv[l], self.sides, self.tau[l], self.bias[l],
                                      self.mass[l], self.cout, self.status)
        rec("calib")
        self.mass_host.copy_(self.mass, non_blocking=True)
        st.synchronize()
        scas = vark.vark_scas_finalize(self.mass_host.numpy())
        keep = vark.vark_build_schedule(scas, self.sides, w.budget_bp, w.n_sinks)
        self.last_scas = scas
        self.keep_host.numpy()[...] = keep
        self.keep.copy_(self.keep_host, non_blocking=True)
        rec("sched")
        vark.vark_build_offsets(self.keep, self.sides, B, D, self.head_off, self.seg_off, self.past_len,
                                self.layer_base)
        self.base_host.copy_(self.layer_base, non_blocking=True)
        rec("offs")
        vark.vark_compact_kv(self.k, self.v, B * H * self.T * D, L, B, H, self.sides, D, self.keep, self.head_off,
                             self.seg_off, self.layer_base, self.kc, self.vc)
        rec("comp")
        st.synchronize()   # layer_base on the host gives each layer's compacted row count
        base = self.base_host.numpy()
        for l in range(L):
            rows = int(base[l + 1] - base[l]) // D
            b0, b1 = int(base[l]), int(base[l + 1])
            vark.vark_pruned_attention(self.q[l], self.kc[b0:b1] if rows else None,
                                       self.vc[b0:b1] if rows else None, rows, self.k[l], self.v[l], self.sides, -1,
                                       self.head_off[l], self.seg_off[l], self.past_len[l], self.tau[l], self.bias[l],
                                       self.out[l], self.status)
        rec("attn")
        self.last_keep = keep
        self.launches += 2 * L + 2
        return keep

    def step_streamed(self, host_in, host_out, cs, ds):
        """One step with its inputs copied in from pinned host buffers and its
        outputs copied back, overlapped with the kernels layer by layer."""
        torch, vark, w = self.torch, self.vark, self.w
        L, B, H, D = w.layers, w.batch, w.heads, w.head_dim
        ms = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(ms)
        ev_cal = [torch.cuda.Event() for _ in range(L)]
        ev_q = [torch.cuda.Event() for _ in range(L)]
        ev_kv, ev_done = torch.cuda.Event(), [torch.cuda.Event() for _ in range(L)]
        cs.wait_event(start)
        with torch.cuda.stream(cs):
            for l in range(L):
                for name in ("cq", "ck", "cv"):
                    getattr(self, name)[l].copy_(host_in[name][l], non_blocking=True)
                ev_cal[l].record(cs)
            for l in range(L):
                self.k[l].copy_(host_in["k"][l], non_blocking=True)
                self.v[l].copy_(host_in["v"][l], non_blocking=True)
            ev_kv.record(cs)
            for l in range(L):
                self.q[l].copy_(host_in["q"][l], non_blocking=True)
                ev_q[l].record(cs)
        self.mass.zero_()
        for l in range(L):
            ms.wait_event(ev_cal[l])
            vark.vark_scas_accumulate(self.cq[l], self.ck[l], self.cv[l], self.sides, self.tau[l], self.bias[l],
                                      self.mass[l], self.cout, self.status)
        self.mass_host.copy_(self.mass, non_blocking=True)
        ms.synchronize()
        scas = vark.vark_scas_finalize(self.mass_host.numpy())
        keep = vark.vark_build_schedule(scas, self.sides, w.budget_bp, w.n_sinks)
        self.keep_host.numpy()[...] = keep
        self.keep.copy_(self.keep_host, non_blocking=True)
        vark.vark_build_offsets(self.keep, self.sides, B, D, self.head_off, self.seg_off, self.past_len,
                                self.layer_base)
        self.base_host.copy_(self.layer_base, non_blocking=True)
        ms.wait_event(ev_kv)
        vark.vark_compact_kv(self.k, self.v, B * H * self.T * D, L, B, H, self.sides, D, self.keep, self.head_off,
                             self.seg_off, self.layer_base, self.kc, self.vc)
        ms.synchronize()
        base = self.base_host.numpy()
        for l in range(L):
            rows = int(base[l + 1] - base[l]) // D
            b0, b1 = int(base[l]), int(base[l + 1])
            ms.wait_event(ev_q[l])
            vark.vark_pruned_attention(self.q[l], self.kc[b0:b1] if rows else None,
                                       self.vc[b0:b1] if rows else None, rows, self.k[l], self.v[l], self.sides, -1,
                                       self.head_off[l], self.seg_off[l], self.past_len[l], self.tau[l], self.bias[l],
                                       self.out[l], self.status)
            ev_done[l].record(ms)
        with torch.cuda.stream(ds):
            for l in range(L):
                ds.wait_event(ev_done[l])
                host_out[l].copy_(self.out[l], non_blocking=True)
        cs.synchronize()
        ds.synchronize()
        ms.synchronize()
        self.launches += 2 * L + 2
        return keep

    def work(self, keep):
        w = self.w
        pf = pruned_flops(keep, self.sides, w.batch, w.head_dim)
        n = np.array([s * s for s in self.sides], dtype=np.int64)
        kept_rows = int((keep.astype(np.int64) * n[None, None, :]).sum())
        comp_bytes = 2.0 * kept_rows * w.batch * w.head_dim * 2 * 2      # read + write, K and V, bf16
        qtok = float(w.layers * w.batch * self.T)
        return {"calib_flops": self.calib_flops, "pruned_flops": pf, "comp_bytes": comp_bytes, "query_tokens": qtok}


def arm_config(w, world):
    """The `config` object of the JSON line (both arms)."""
    return {"workload": WORKLOAD + ": 32 layers x 16 heads, head_dim 128, 1024^2 scales (10,521 tokens), "
                                   "batch 8, budget 10%, sinks 0-1, calibration 16 seeds per layer",
            "global_batch": w.batch * world, "seq_len": synth.n_tokens(w.sides),
            "parallelism": f"replicas x{world}", "l2": "inputs larger than L2 (no flush needed)",
            "value_def": "(calibration + pruned attention FLOPs) / step time; step = calibration, "
                         "S-CAS, schedule, offsets, compaction, pruned attention of all layers"}


def reference_arm(args, rank, world):
    """The oracle, as it stands, on the host cores: bounded samples of the
    workload per step."""
    if rank != 0:
        return 0
    from threadpoolctl import threadpool_info
    w = synth.WORKLOADS[WORKLOAD]
    sample = CpuSample(w)
    for _ in range(args.warmup):
        sample.run(small=True)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += sample.run()
    dt = time.perf_counter() - t0
    val = flops / dt / 1e12
    cores = max([x.get("num_threads", 1) for x in threadpool_info()] or [1])
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(w, world),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample.describe(), "per_step": sample.per_step()},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


class CpuSample:
    """A bounded slice of one step for the oracle, each part timed on its own
    and reported in the GPU path's unit for that part:

    * calibration attention of one seed and one head of one layer at full T
      (TFLOP/s);
    * S-CAS finalisation + schedule of all 32 layers (in full, ms);
    * offsets of all 32 layers (in full, ms);
    * compaction of one (layer, batch) element (GB/s, read + write);
    * pruned attention of two heads of one batch element of one layer
      (TFLOP/s and query tokens/s).

    Full-step seconds are extrapolated linearly from each slice by the
    algorithmic work ratio and labelled so."""

    def __init__(self, w):
        import oracle
        self.o = oracle
        self.w = w
        self.sides = w.sides
        self.g = oracle.ScaleGeometry(w.sides)
        T, D, H, S = self.g.T, w.head_dim, w.heads, self.g.S
        key = synth.derive_key(w.base_seed, 0xC0)
        f = lambda bits: (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
        self.qkv = [f(synth.normal_bf16_bits(synth.derive_key(key, i), (1, 2, T, D))) for i in range(3)]
        self.kbits = synth.normal_bf16_bits(synth.derive_key(key, 7), (1, 1, H, T, D))
        self.vbits = synth.normal_bf16_bits(synth.derive_key(key, 8), (1, 1, H, T, D))
        self.tau = synth.gen_tau(key, H).astype(np.float64)
        self.bias = synth.gen_bias(key, H, S).astype(np.float64)
        self.M = np.random.default_rng(1).uniform(0, 1, size=(w.layers, H, S, S))
        self.t = {k: 0.0 for k in ("calibration", "schedule", "offsets", "compaction", "pruned_attention")}
        self.work = {k: 0.0 for k in self.t}
        self.full = None

    def describe(self):
        return ("oracle fp64 slice per step: calibration attention of 1 seed x 1 head x 1 layer at full T, "
                "S-CAS + schedule + offsets of all 32 layers, compaction of 1 (layer, batch), pruned attention of "
                "1 batch x 2 heads x 1 layer; FLOPs counted as on the GPU")

    def run(self, small=False):
        """One slice; returns its attention FLOPs (calibration + pruned)."""
        o, w, g = self.o, self.w, self.g
        D = w.head_dim
        q, k, v = self.qkv
        tic = time.perf_counter()
        o.block_causal_attention(q[:, :1], k[:, :1], v[:, :1], self.sides, self.tau[:1], self.bias[:1])
        cf = calib_flops(self.sides, 1, 1, D)
        if small:
            return cf
        self.t["calibration"] += time.perf_counter() - tic
        self.work["calibration"] += cf
        tic = time.perf_counter()
        scas = o.scas_from_mass(self.M)
        keep = o.build_schedule(scas, self.sides, w.budget_bp, w.n_sinks)
        self.t["schedule"] += time.perf_counter() - tic
        self.work["schedule"] += 1
        tic = time.perf_counter()
        o.build_offsets(keep, self.sides, w.batch, D)
        self.t["offsets"] += time.perf_counter() - tic
        self.work["offsets"] += 1
        k1 = keep[:1]
        ho1, so1, pl1, lb1 = o.build_offsets(k1, self.sides, 1, D)
        tic = time.perf_counter()
        o.compact_kv(self.kbits, self.vbits, k1, self.sides, ho1, so1, lb1)
        self.t["compaction"] += time.perf_counter() - tic
        self.work["compaction"] += 2.0 * int(lb1[-1]) * 2 * 2          # read + write, K and V, bf16
        kd = (self.kbits[0].astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
        vd = (self.vbits[0].astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
        tic = time.perf_counter()
        o.pruned_attention(q[:, :2], kd[:, :2], vd[:, :2], keep[0, :2], self.sides, self.tau[:2], self.bias[:2])
        self.t["pruned_attention"] += time.perf_counter() - tic
        pf = pruned_flops(keep[:1, :2], self.sides, 1, D)
        self.work["pruned_attention"] += pf
        if self.full is None:
            n = np.array([x * x for x in self.sides], dtype=np.int64)
            kept = int((keep.astype(np.int64) * n[None, None, :]).sum())
            self.full = {"calibration": calib_flops(self.sides, w.n_seeds, w.heads, D) * w.layers,
                         "compaction": 2.0 * kept * w.batch * D * 2 * 2,
                         "pruned_attention": pruned_flops(keep, self.sides, w.batch, D),
                         "query_tokens": float(w.layers * w.batch * g.T)}
        return cf + pf

    def per_step(self):
        """Each part's rate in the GPU path's unit, with the full-step seconds
        extrapolated from the slice."""
        t, wk, full = self.t, self.work, self.full
        if not full or t["calibration"] <= 0:
            return None
        reps = wk["schedule"]
        g = self.g
        q_rows_slice = 2.0 * g.T                # 2 heads x all query rows of one batch element
        out = {
            "calibration_attention": {
                "tflops": wk["calibration"] / t["calibration"] / 1e12,
                "sample": "1 seed x 1 head x 1 layer, full T",
                "full_step_s_extrapolated": full["calibration"] / (wk["calibration"] / t["calibration"]),
                "scaling": "linear in algorithmic FLOPs (x%d)" % round(full["calibration"] / (wk["calibration"] / reps))},
            "scas_finalise_and_schedule": {"ms": t["schedule"] / reps * 1e3, "sample": "all 32 layers (full)"},
            "offsets": {"ms": t["offsets"] / reps * 1e3, "sample": "all 32 layers (full)"},
            "compaction": {
                "gbs": wk["compaction"] / t["compaction"] / 1e9,
                "sample": "1 (layer, batch) element of the 32 x 8",
                "full_step_s_extrapolated": full["compaction"] / (wk["compaction"] / t["compaction"]),
                "scaling": "linear in bytes moved"},
            "pruned_attention": {
                "tflops": wk["pruned_attention"] / t["pruned_attention"] / 1e12,
                "query_tokens_per_s": q_rows_slice * reps / t["pruned_attention"],
                "sample": "1 batch element x 2 heads x 1 layer, all 13 query scales",
                "full_step_s_extrapolated": full["pruned_attention"] / (wk["pruned_attention"] / t["pruned_attention"]),
                "scaling": "linear in algorithmic FLOPs"},
        }
        out["full_step_s_extrapolated"] = (out["calibration_attention"]["full_step_s_extrapolated"]
                                           + out["compaction"]["full_step_s_extrapolated"]
                                           + out["pruned_attention"]["full_step_s_extrapolated"]
                                           + (t["schedule"] + t["offsets"]) / reps)
        return out


def int8_cache(pipe, max_over_ranks, bf16_attention_ms, hbm_gbs, reps=3):
    """The retained cache stored as int8 codes with per-(block, channel) absmax:
    quantising compaction of all layers, then per layer either dequantisation
    into a one-layer bf16 buffer followed by that layer's pruned attention, or
    pruned attention straight over the codes (dequantised in the kernel)."""
    import torch
    vark, w = pipe.vark, pipe.w
    L, B, H, D, S, T = w.layers, w.batch, w.heads, w.head_dim, pipe.S, pipe.T
    base = pipe.base_host.numpy()
    total = int(base[-1])
    dev = pipe.dev
    kq = torch.empty(max(total, 16), dtype=torch.int8, device=dev)
    vq = torch.empty_like(kq)
    ka = torch.empty((L, B, H, S, D), dtype=torch.float32, device=dev)
    va = torch.empty_like(ka)
    max_rows = max(int(base[l + 1] - base[l]) // D for l in range(L))
    kcl = torch.empty(max(max_rows * D, 16), dtype=torch.bfloat16, device=dev)
    vcl = torch.empty_like(kcl)
    st = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]

    def one():
        ev[0].record(st)
        vark.vark_quantize_kv_int8(pipe.k, pipe.v, B * H * T * D, L, B, H, pipe.sides, D, pipe.keep, pipe.head_off,
                                   pipe.seg_off, pipe.layer_base, kq, vq, ka, va)
        ev[1].record(st)
        for l in range(L):
            rows = int(base[l + 1] - base[l]) // D
            b0 = int(base[l])
            vark.vark_dequantize_layer_int8(kq[b0:], vq[b0:], ka[l], va[l], rows, B, H, pipe.sides, D,
                                            pipe.head_off[l], pipe.seg_off[l], kcl, vcl)
            vark.vark_pruned_attention(pipe.q[l], kcl if rows else None, vcl if rows else None, rows, pipe.k[l],
                                       pipe.v[l], pipe.sides, -1, pipe.head_off[l], pipe.seg_off[l],
                                       pipe.past_len[l], pipe.tau[l], pipe.bias[l], pipe.out[l], pipe.status)
        ev[2].record(st)
        for l in range(L):     # the dequantisations alone
            rows = int(base[l + 1] - base[l]) // D
            b0 = int(base[l])
            vark.vark_dequantize_layer_int8(kq[b0:], vq[b0:], ka[l], va[l], rows, B, H, pipe.sides, D,
                                            pipe.head_off[l], pipe.seg_off[l], kcl, vcl)
        ev[3].record(st)
        for l in range(L):     # attention straight over the codes
            rows = int(base[l + 1] - base[l]) // D
            b0 = int(base[l])
            vark.vark_pruned_attention_int8(pipe.q[l], kq[b0:], vq[b0:], ka[l], va[l], rows, pipe.k[l], pipe.v[l],
                                            pipe.sides, -1, pipe.head_off[l], pipe.seg_off[l], pipe.past_len[l],
                                            pipe.tau[l], pipe.bias[l], pipe.out[l], pipe.status)
        ev[4].record(st)

    one()
    torch.cuda.synchronize()
    tq = ta = td = tf = 0.0
    for _ in range(reps):
        one()
        torch.cuda.synchronize()
        tq += ev[0].elapsed_time(ev[1]) / 1e3
        ta += ev[1].elapsed_time(ev[2]) / 1e3
        td += ev[2].elapsed_time(ev[3]) / 1e3
        tf += ev[3].elapsed_time(ev[4]) / 1e3
    assert int(pipe.status.item()) == 0
    tq, ta, td = max_over_ranks(tq / reps), max_over_ranks(ta / reps), max_over_ranks(td / reps)
    tf = max_over_ranks(tf / reps)
    bf16_bytes = 2 * 2 * total
    absmax_bytes = 2 * 4 * ka.numel()
    int8_bytes = 2 * total + absmax_bytes
    # algorithmic bytes: quantise = kept bf16 K,V read once + codes and absmax tables written;
    # dequantise = codes and absmax read + bf16 K,V written
    q_bytes = bf16_bytes + int8_bytes
    return {"cache_bytes_bf16": bf16_bytes, "cache_bytes_int8": int8_bytes,
            "cache_ratio": int8_bytes / bf16_bytes, "quantize_ms": tq * 1e3,
            "quantize_gbs": q_bytes / tq / 1e9, "quantize_frac_of_hbm": q_bytes / tq / 1e9 / hbm_gbs,
            "dequantize_ms": td * 1e3, "dequantize_gbs": q_bytes / td / 1e9,
            "dequantize_frac_of_hbm": q_bytes / td / 1e9 / hbm_gbs,
            "dequant_plus_attention_ms": ta * 1e3, "fused_attention_ms": tf * 1e3,
            "bf16_cache_attention_ms": bf16_attention_ms}


def packed_cache(pipe, max_over_ranks, bf16_attention_ms, hbm_gbs, bits, reps=3):
    """The retained cache stored as packed 4-bit or 3-bit codes with
    per-(block, channel) bf16 scales: quantising compaction of all layers,
    then per layer either dequantisation into a one-layer bf16 buffer followed
    by that layer's pruned attention, or pruned attention straight over the
    codes (dequantised in the kernel)."""
    import torch
    vark, w = pipe.vark, pipe.w
    L, B, H, D, S, T = w.layers, w.batch, w.heads, w.head_dim, pipe.S, pipe.T
    num, den = {4: (1, 2), 3: (3, 8)}[bits]      # code bytes per element
    quantize = {4: vark.vark_quantize_kv_int4, 3: vark.vark_quantize_kv_int3}[bits]
    dequantize = {4: vark.vark_dequantize_layer_int4, 3: vark.vark_dequantize_layer_int3}[bits]
    fused = {4: vark.vark_pruned_attention_int4, 3: vark.vark_pruned_attention_int3}[bits]
    base = pipe.base_host.numpy()
    total = int(base[-1])
    dev = pipe.dev
    kq = torch.empty(max(num * total // den, 16), dtype=torch.uint8, device=dev)
    vq = torch.empty_like(kq)
    ks = torch.empty((L, B, H, S, D), dtype=torch.int16, device=dev)
    vs = torch.empty_like(ks)
    max_rows = max(int(base[l + 1] - base[l]) // D for l in range(L))
    kcl = torch.empty(max(max_rows * D, 16), dtype=torch.bfloat16, device=dev)
    vcl = torch.empty_like(kcl)
    st = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]

    def one():
        ev[0].record(st)
        quantize(pipe.k, pipe.v, B * H * T * D, L, B, H, pipe.sides, D, pipe.keep, pipe.head_off, pipe.seg_off,
                 pipe.layer_base, kq, vq, ks, vs)
        ev[1].record(st)
        for l in range(L):
            rows = int(base[l + 1] - base[l]) // D
            b0 = num * int(base[l]) // den
            dequantize(kq[b0:], vq[b0:], ks[l], vs[l], rows, B, H, pipe.sides, D, pipe.head_off[l],
                       pipe.seg_off[l], kcl, vcl)
            vark.vark_pruned_attention(pipe.q[l], kcl if rows else None, vcl if rows else None, rows, pipe.k[l],
                                       pipe.v[l], pipe.sides, -1, pipe.head_off[l], pipe.seg_off[l],
                                       pipe.past_len[l], pipe.tau[l], pipe.bias[l], pipe.out[l], pipe.status)
        ev[2].record(st)
        for l in range(L):     # the dequantisations alone
            rows = int(base[l + 1] - base[l]) // D
            b0 = num * int(base[l]) // den
            dequantize(kq[b0:], vq[b0:], ks[l], vs[l], rows, B, H, pipe.sides, D, pipe.head_off[l],
                       pipe.seg_off[l], kcl, vcl)
        ev[3].record(st)
        for l in range(L):     # attention straight over the codes
            rows = int(base[l + 1] - base[l]) // D
            b0 = num * int(base[l]) // den
            fused(pipe.q[l], kq[b0:], vq[b0:], ks[l], vs[l], rows, pipe.k[l], pipe.v[l], pipe.sides, -1,
                  pipe.head_off[l], pipe.seg_off[l], pipe.past_len[l], pipe.tau[l], pipe.bias[l], pipe.out[l],
                  pipe.status)
        ev[4].record(st)

    one()
    torch.cuda.synchronize()
    tq = ta = td = tf = 0.0
    for _ in range(reps):
        one()
        torch.cuda.synchronize()
        tq += ev[0].elapsed_time(ev[1]) / 1e3
        ta += ev[1].elapsed_time(ev[2]) / 1e3
        td += ev[2].elapsed_time(ev[3]) / 1e3
        tf += ev[3].elapsed_time(ev[4]) / 1e3
    assert int(pipe.status.item()) == 0
    tq, ta, td = max_over_ranks(tq / reps), max_over_ranks(ta / reps), max_over_ranks(td / reps)
    tf = max_over_ranks(tf / reps)
    bf16_bytes = 2 * 2 * total
    packed_bytes = 2 * (num * total // den) + 2 * 2 * ks.numel()
    q_bytes = bf16_bytes + packed_bytes   # kept bf16 K, V read once; packed codes and scale tables written
    return {"cache_bytes_bf16": bf16_bytes, f"cache_bytes_int{bits}": packed_bytes,
            "cache_ratio": packed_bytes / bf16_bytes,
            "quantize_ms": tq * 1e3, "quantize_gbs": q_bytes / tq / 1e9,
            "quantize_frac_of_hbm": q_bytes / tq / 1e9 / hbm_gbs,
            "dequantize_ms": td * 1e3, "dequantize_gbs": q_bytes / td / 1e9,
            "dequantize_frac_of_hbm": q_bytes / td / 1e9 / hbm_gbs,
            "dequant_plus_attention_ms": ta * 1e3, "fused_attention_ms": tf * 1e3,
            "bf16_cache_attention_ms": bf16_attention_ms}


def scas_only(pipe, max_over_ranks, with_o_ms, peaks, reps=2):
    """Calibration of every layer called without an output buffer (S-CAS
    only: the kernel skips V and the PV MMAs), timed with CUDA events outside
    the step.  Algorithmic work here is the QK^T half of the calibration
    FLOPs."""
    import torch
    vark, w = pipe.vark, pipe.w
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def run():
        pipe.mass.zero_()
        for l in range(w.layers):
            vark.vark_scas_accumulate(pipe.cq[l], pipe.ck[l], pipe.cv[l], pipe.sides, pipe.tau[l], pipe.bias[l],
                                      pipe.mass[l], None, pipe.status)
    run()
    torch.cuda.synchronize()
    t = 0.0
    for _ in range(reps):
        e0.record(st)
        run()
        e1.record(st)
        torch.cuda.synchronize()
        t += e0.elapsed_time(e1) / 1e3
    assert int(pipe.status.item()) == 0
    t = max_over_ranks(t / reps)
    qk = pipe.calib_flops / 2
    return {"ms_per_step": t * 1e3, "with_output_ms_per_step": with_o_ms, "speedup": with_o_ms / (t * 1e3),
            "qk_tflops": qk / t / 1e12, "qk_frac_of_bf16_peak": qk / t / 1e12 / peaks["bf16_tflops_sustained"],
            "note": "all 32 layers, 16 seeds each; FLOPs = the QK^T half of the calibration work"}


def ranking_stability(pipe):
    """S-CAS of every layer from two disjoint halves of the calibration seeds,
    compared by vark_rank_stability (Spearman over candidate pairs, Jaccard of
    the two schedules' drop sets at the workload's budget)."""
    import torch
    vark, w = pipe.vark, pipe.w
    L, H, S = w.layers, w.heads, pipe.S
    half = w.n_seeds // 2
    ma = torch.zeros((L, H, S, S), dtype=torch.float32, device=pipe.dev)
    mb = torch.zeros_like(ma)
    t0 = time.perf_counter()
    for l in range(L):
        vark.vark_scas_accumulate(pipe.cq[l][:half], pipe.ck[l][:half], pipe.cv[l][:half], pipe.sides, pipe.tau[l],
                                  pipe.bias[l], ma[l], None, pipe.status)
        vark.vark_scas_accumulate(pipe.cq[l][half:], pipe.ck[l][half:], pipe.cv[l][half:], pipe.sides, pipe.tau[l],
                                  pipe.bias[l], mb[l], None, pipe.status)
    torch.cuda.synchronize()
    assert int(pipe.status.item()) == 0
    sa = vark.vark_scas_finalize(ma.cpu().numpy())
    sb = vark.vark_scas_finalize(mb.cpu().numpy())
    sp, jc = vark.vark_rank_stability(sa, sb, pipe.sides, w.budget_bp, w.n_sinks)
    return {"seeds": f"{half} vs {w.n_seeds - half} (disjoint)", "spearman": sp, "drop_jaccard": jc,
            "budget_bp": w.budget_bp, "seconds": time.perf_counter() - t0}


def other_configs(rank, device, max_over_ranks, peaks, reps=3):
    """The two other 1024^2 workloads, timed per kernel with CUDA events
    (outside the benchmark step):
    - large_8l: 8 layers x 32 heads, batch 4, 4% budget, 8 calibration seeds:
      calibration attention, compaction and pruned attention of all layers;
    - final_scale: the 64x64 scale's 4,096 queries against the 10,521-token
      cache, budgets {100, 20, 10, 4}% x batch {1, 4, 16, 32}, seed-random
      retained sets per head; L2 flushed (1 GiB written) before each of 10
      timed launches (the small-batch inputs fit in L2).
    The 8-layer compaction is also timed alone, 10 launches back to back
    between one pair of events (its 0.44 GB exceed L2)."""
    import torch
    import kv_cache_compression_cas_b200 as vark
    res = {}
    st = torch.cuda.current_stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]

    # ---- large_8l
    w = synth.WORKLOADS["large_8l"]
    pipe = Pipeline(w, rank, device)
    ph = {"calib": 0.0, "comp": 0.0, "attn": 0.0}
    keys = ("t0", "calib", "sched", "offs", "comp", "attn")
    ev = dict(zip(keys, evs))
    pipe.step()
    torch.cuda.synchronize()
    for _ in range(reps):
        pipe.step(ev)
        torch.cuda.synchronize()
        ph["calib"] += ev["t0"].elapsed_time(ev["calib"]) / 1e3
        ph["comp"] += ev["offs"].elapsed_time(ev["comp"]) / 1e3
        ph["attn"] += ev["comp"].elapsed_time(ev["attn"]) / 1e3
    assert int(pipe.status.item()) == 0
    for k_ in ph:
        ph[k_] = max_over_ranks(ph[k_] / reps)
    keep = pipe.last_keep
    base = pipe.base_host.numpy()
    comp_bytes = 2 * 2 * 2 * int(base[-1])
    pf = pruned_flops(keep, w.sides, w.batch, w.head_dim)
    # The compaction kernel alone: at 0.44 GB it runs for ~0.1 ms, so the
    # host's call overhead between the step's events is a visible share of the
    # in-step interval.  Here n_back launches go back to back between one pair
    # of events (the host stays ahead of the GPU); the bytes moved per launch
    # (0.22 GB read, 0.22 GB written) exceed L2, so no flush is needed.
    L8, B8, H8, D8, T8 = w.layers, w.batch, w.heads, w.head_dim, pipe.T

    def compact8():
        vark.vark_compact_kv(pipe.k, pipe.v, B8 * H8 * T8 * D8, L8, B8, H8, w.sides, D8, pipe.keep, pipe.head_off,
                             pipe.seg_off, pipe.layer_base, pipe.kc, pipe.vc)
    n_back = 10
    compact8()
    torch.cuda.synchronize()
    evs[0].record(st)
    for _ in range(n_back):
        compact8()
    evs[1].record(st)
    torch.cuda.synchronize()
    ck = max_over_ranks(evs[0].elapsed_time(evs[1]) / 1e3 / n_back)
    res["large_8l"] = {
        "workload": "8 layers x 32 heads, head_dim 128, 1024^2 scales, batch 4, budget 4%, 8 calibration seeds",
        "calibration_tflops": pipe.calib_flops / ph["calib"] / 1e12,
        "calibration_frac_of_bf16_peak": pipe.calib_flops / ph["calib"] / 1e12 / peaks["bf16_tflops_sustained"],
        "compaction_gbs": comp_bytes / ph["comp"] / 1e9,
        "compaction_frac_of_hbm": comp_bytes / ph["comp"] / 1e9 / peaks["hbm_gbs"],
        "compaction_kernel_gbs": comp_bytes / ck / 1e9,
        "compaction_kernel_frac_of_hbm": comp_bytes / ck / 1e9 / peaks["hbm_gbs"],
        "pruned_attention_tflops": pf / ph["attn"] / 1e12,
        "pruned_frac_of_bf16_peak": pf / ph["attn"] / 1e12 / peaks["bf16_tflops_sustained"],
        "query_tokens_per_s": w.layers * w.batch * pipe.T / ph["attn"],
        "ms": {k_: v_ * 1e3 for k_, v_ in ph.items()}}
    del pipe
    torch.cuda.empty_cache()

    # ---- final_scale sweep
    w = synth.WORKLOADS["final_scale"]
    sides, H, D, kq = w.sides, w.heads, w.head_dim, w.query_scale
    S, T = len(sides), synth.n_tokens(sides)
    n = [x * x for x in sides]
    # 1 GiB flush: writing it also keeps the GPU busy for longer than the
    # host's call overhead, so that overhead stays outside the timed launch
    flush = torch.empty(1 << 30, dtype=torch.uint8, device=device)
    sweep_reps = max(reps, 10)
    tau = torch.from_numpy(synth.gen_tau(w.base_seed, H)).to(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    rows = []
    for B in w.extra["batches"]:
        seed = synth.derive_key(w.base_seed, 0xF5, B, rank)
        q = randn_bf16((B, H, n[kq], D), seed + 1, device)
        kd = randn_bf16((B, H, T, D), seed + 2, device)
        vd = randn_bf16((B, H, T, D), seed + 3, device)
        out = torch.empty_like(q)
        for budget in w.extra["budgets_bp"]:
            keep = synth.random_keep(synth.derive_key(w.base_seed, budget), H, sides, budget, w.n_sinks, kq)
            keep_d = torch.from_numpy(keep).to(device)
            ho = torch.empty((1, H), dtype=torch.int32, device=device)
            so = torch.empty((1, H, S), dtype=torch.int32, device=device)
            pl = torch.empty((1, H, S), dtype=torch.int32, device=device)
            lb = torch.empty(2, dtype=torch.int64, device=device)
            vark.vark_build_offsets(keep_d, sides, B, D, ho, so, pl, lb)
            total = int(lb[-1].item())
            kc = torch.empty(max(total, 16), dtype=torch.bfloat16, device=device)
            vc = torch.empty_like(kc)
            vark.vark_compact_kv(kd[None], vd[None], B * H * T * D, 1, B, H, sides, D, keep_d, ho, so, lb, kc, vc)

            def launch():
                vark.vark_pruned_attention(q, kc if total else None, vc if total else None, total // D, kd, vd,
                                           sides, kq, ho[0], so[0], pl[0], tau, None, out, status)
            for _ in range(2):
                launch()
            t = 0.0
            for _ in range(sweep_reps):
                flush.fill_(1)
                evs[0].record(st)
                launch()
                evs[1].record(st)
                torch.cuda.synchronize()
                t += evs[0].elapsed_time(evs[1]) / 1e3
            t = max_over_ranks(t / sweep_reps)
            assert int(status.item()) == 0
            past = (keep[0, :, :kq].astype(np.float64) * np.array(n[:kq], dtype=np.float64)).sum(axis=1)
            fl = float((4.0 * B * n[kq] * (past + n[kq]) * D).sum())
            rows.append({"budget_bp": budget, "batch": B, "tflops": fl / t / 1e12,
                         "frac_of_bf16_peak": fl / t / 1e12 / peaks["bf16_tflops"],
                         "frac_of_sustained_bf16_peak": fl / t / 1e12 / peaks["bf16_tflops_sustained"],
                         "query_tokens_per_s": B * n[kq] / t, "ms": t * 1e3})
        del q, kd, vd, out
    res["final_scale"] = {"workload": "query scale 12 (4,096 rows) vs the 10,521-token cache, 16 heads, head_dim 128; "
                                      "fractions against the burst and the sustained bf16 peak (10 launches, L2 flushed before "
                                      "each; batch-32 launches of 5-11 ms run power-capped)", "points": rows}
    del flush
    torch.cuda.empty_cache()
    return res


def generation_order(pipe, passes, max_over_ranks, sum_over_ranks):
    """The inference flow scale by scale on the same workload and schedule:
    for each scale k, pruned attention of scale k's queries in every layer over
    the cache appended so far plus scale k itself, then the append of scale k
    for all layers.  Returns its throughput next to the one-shot path's."""
    import torch
    vark, w = pipe.vark, pipe.w
    L, B, H, D = w.layers, w.batch, w.heads, w.head_dim
    sides = pipe.sides
    n = [s * s for s in sides]
    off = np.cumsum([0] + n[:-1])
    per_scale = []
    for k in range(len(sides)):
        sl = slice(int(off[k]), int(off[k]) + n[k])
        per_scale.append((pipe.q[:, :, :, sl].contiguous(), pipe.k[:, :, :, sl].contiguous(),
                          pipe.v[:, :, :, sl].contiguous()))
    keep = pipe.last_keep
    base = pipe.base_host.numpy()
    st = torch.cuda.current_stream()
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(sides) * passes + 2)]
    outs = [torch.empty_like(t[0]) for t in per_scale]

    def one_pass(evs):
        pipe.kc.zero_()
        pipe.vc.zero_()
        for k, (qk, kk, vk) in enumerate(per_scale):
            if evs is not None:
                evs[2 * k].record(st)
            for l in range(L):
                rows = int(base[l + 1] - base[l]) // D
                b0, b1 = int(base[l]), int(base[l + 1])
                vark.vark_pruned_attention_step(qk[l], pipe.kc[b0:b1] if rows else None,
                                                pipe.vc[b0:b1] if rows else None, rows, kk[l], vk[l], sides, k,
                                                pipe.head_off[l], pipe.seg_off[l], pipe.past_len[l], pipe.tau[l],
                                                pipe.bias[l], outs[k][l], pipe.status)
            if evs is not None:
                evs[2 * k + 1].record(st)
            vark.vark_append_scale(kk, vk, B * H * n[k] * D, L, B, H, sides, D, k, pipe.keep, pipe.head_off,
                                   pipe.seg_off, pipe.layer_base, pipe.kc, pipe.vc)

    one_pass(None)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    attn_s = 0.0
    e0.record(st)
    for i in range(passes):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(sides))]
        one_pass(evs)
        torch.cuda.synchronize()
        attn_s += sum(evs[2 * k].elapsed_time(evs[2 * k + 1]) for k in range(len(sides))) / 1e3
    e1.record(st)
    torch.cuda.synchronize()
    assert int(pipe.status.item()) == 0
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    attn_s = max_over_ranks(attn_s)
    fl = pruned_flops(keep, sides, B, D) * passes
    nl = np.array(n, dtype=np.int64)
    kept_rows = int((keep.astype(np.int64) * nl[None, None, :]).sum())
    app_bytes = 2.0 * kept_rows * B * D * 2 * 2 * passes
    static = {"passes": passes, "ms_per_pass": t * 1e3 / passes,
              "attention_tflops": sum_over_ranks(fl) / attn_s / 1e12,
              "append_and_zero_ms_per_pass": (t - attn_s) * 1e3 / passes,
              "query_tokens_per_s": sum_over_ranks(float(L * B * pipe.T * passes)) / t,
              "append_bytes_per_pass": app_bytes / passes,
              "peak_cache_bytes": 4 * int(base[-1]),
              "launches_per_pass": len(sides) * (L + 1) + 2}
    return {"static_schedule": static,
            "early_pruning": early_pruning_order(pipe, per_scale, outs, passes, max_over_ranks, sum_over_ranks)}


def early_pruning_order(pipe, per_scale, outs, passes, max_over_ranks, sum_over_ranks):
    """Scale by scale under the time-varying schedule (BINARY-HEATKV with
    GREEDYEARLYPRUNING, the library's reading) at the same absolute budget:
    attention over the cache held after the previous step, then the survivors
    move to the new layout and the new scale is appended."""
    import torch
    vark, w = pipe.vark, pipe.w
    L, B, H, D, S = w.layers, w.batch, w.heads, w.head_dim, pipe.S
    sides = pipe.sides
    n = np.array([s * s for s in sides], dtype=np.int64)
    prefix, evict = vark.vark_build_early_pruning_schedule(pipe.last_scas, sides, w.budget_bp, w.n_sinks)
    idx = np.arange(S)[None, None, :]
    keeps = [((idx <= k) & (evict.astype(np.int64) > k)).astype(np.uint8) for k in range(S)]
    held = [int((kp * n[None, None, :]).sum()) for kp in keeps]
    cap = B * D * (max(held) + int(n.max()) + 1)
    dev = pipe.dev
    bufs = [(torch.zeros(cap, dtype=torch.bfloat16, device=dev), torch.zeros(cap, dtype=torch.bfloat16, device=dev))
            for _ in range(2)]
    tabs = []
    for k in range(S):                               # tables of every step's retained set (schedule data)
        kp = torch.from_numpy(keeps[k]).to(dev)
        t = {"keep": kp, "head_off": torch.empty((L, H), dtype=torch.int32, device=dev),
             "seg_off": torch.empty((L, H, S), dtype=torch.int32, device=dev),
             "past_len": torch.empty((L, H, S), dtype=torch.int32, device=dev),
             "layer_base": torch.empty(L + 1, dtype=torch.int64, device=dev)}
        vark.vark_build_offsets(kp, sides, B, D, t["head_off"], t["seg_off"], t["past_len"], t["layer_base"])
        t["base"] = t["layer_base"].cpu().numpy()
        tabs.append(t)
    empty = {"keep": torch.zeros((L, H, S), dtype=torch.uint8, device=dev)}
    for key in ("head_off",):
        empty[key] = torch.zeros((L, H), dtype=torch.int32, device=dev)
    empty["seg_off"] = torch.full((L, H, S), -1, dtype=torch.int32, device=dev)
    empty["past_len"] = torch.zeros((L, H, S), dtype=torch.int32, device=dev)
    empty["layer_base"] = torch.zeros(L + 1, dtype=torch.int64, device=dev)
    empty["base"] = np.zeros(L + 1, dtype=np.int64)
    st = torch.cuda.current_stream()
    moved = 0

    def one_pass():
        nonlocal moved
        moved = 0
        prev, (kcp, vcp) = empty, bufs[1]
        for k, (qk, kk, vk) in enumerate(per_scale):
            for l in range(L):
                rows = int(prev["base"][l + 1] - prev["base"][l]) // D
                b0, b1 = int(prev["base"][l]), int(prev["base"][l + 1])
                vark.vark_pruned_attention_step(qk[l], kcp[b0:b1] if rows else None, vcp[b0:b1] if rows else None,
                                                rows, kk[l], vk[l], sides, k, prev["head_off"][l],
                                                prev["seg_off"][l], prev["past_len"][l], pipe.tau[l], pipe.bias[l],
                                                outs[k][l], pipe.status)
            t = tabs[k]
            kcn, vcn = bufs[k % 2]
            vark.vark_recompact_kv(kcp, vcp, prev["head_off"], prev["seg_off"], prev["layer_base"], L, B, H, sides,
                                   D, k, t["keep"], t["head_off"], t["seg_off"], t["layer_base"], kcn, vcn)
            vark.vark_append_scale(kk, vk, B * H * int(n[k]) * D, L, B, H, sides, D, k, t["keep"], t["head_off"],
                                   t["seg_off"], t["layer_base"], kcn, vcn)
            moved += 2 * 2 * 2 * int(t["base"][-1])   # read + write, K and V, bf16 (survivors + appended rows)
            prev, (kcp, vcp) = t, (kcn, vcn)

    one_pass()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(passes):
        one_pass()
    e1.record(st)
    torch.cuda.synchronize()
    assert int(pipe.status.item()) == 0
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    nl = n.astype(np.float64)
    fl = 0.0
    for k in range(S):
        kp = keeps[k - 1] if k > 0 else np.zeros_like(keeps[0])
        past = (kp[:, :, :k].astype(np.float64) * nl[None, None, :k]).sum(axis=2)
        fl += float((4.0 * B * nl[k] * (past + nl[k]) * D).sum())
    return {"passes": passes, "ms_per_pass": t * 1e3 / passes,
            "attention_tflops_incl_moves": sum_over_ranks(fl * passes) / t / 1e12,
            "query_tokens_per_s": sum_over_ranks(float(L * B * pipe.T * passes)) / t,
            "prefix_len": [int(x) for x in prefix],
            "peak_cache_bytes": 4 * B * D * max(held), "final_cache_bytes": 4 * B * D * held[-1],
            "bytes_moved_per_pass": moved}


def summarize_kernels(kernels, quant, quant4, quant3, others, scas_o, peaks):
    """Rounded per-kernel rates and roofline fractions (sustained / burst)."""
    bs, bb, hb = peaks["bf16_tflops_sustained"], peaks["bf16_tflops"], peaks["hbm_gbs"]
    r = lambda x: None if x is None else round(float(x), 3)
    out = {"calibration_tflops": r(kernels["scas_calibration_attention"]["tflops"]),
           "calibration_frac": [r(kernels["scas_calibration_attention"]["tflops"] / bs),
                                r(kernels["scas_calibration_attention"]["tflops"] / bb)],
           "pruned_tflops": r(kernels["pruned_attention"]["tflops"]),
           "pruned_frac": [r(kernels["pruned_attention"]["tflops"] / bs), r(kernels["pruned_attention"]["tflops"] / bb)],
           "pruned_query_tokens_per_s": r(kernels["pruned_attention"]["query_tokens_per_s"]),
           "compaction_gbs": r(kernels["compaction"]["gbs"]), "compaction_frac_of_hbm": r(kernels["compaction"]["gbs"] / hb),
           "fractions": "[of sustained, of burst] bf16 peak"}
    if scas_o:
        out["scas_only_qk_tflops"] = r(scas_o["qk_tflops"])
    if quant:
        out["int8"] = {"cache_ratio": r(quant["cache_ratio"]), "quantize_frac_of_hbm": r(quant["quantize_frac_of_hbm"]),
                       "dequantize_frac_of_hbm": r(quant["dequantize_frac_of_hbm"]),
                       "dequant_plus_attention_vs_bf16": r(quant["dequant_plus_attention_ms"] / quant["bf16_cache_attention_ms"]),
                       "fused_attention_vs_bf16": r(quant["fused_attention_ms"] / quant["bf16_cache_attention_ms"])}
    if quant4:
        out["int4"] = {"cache_ratio": r(quant4["cache_ratio"]), "quantize_frac_of_hbm": r(quant4["quantize_frac_of_hbm"]),
                       "dequantize_frac_of_hbm": r(quant4["dequantize_frac_of_hbm"]),
                       "dequant_plus_attention_vs_bf16": r(quant4["dequant_plus_attention_ms"] / quant4["bf16_cache_attention_ms"]),
                       "fused_attention_vs_bf16": r(quant4["fused_attention_ms"] / quant4["bf16_cache_attention_ms"])}
    if quant3:
        out["int3"] = {"cache_ratio": r(quant3["cache_ratio"]), "quantize_frac_of_hbm": r(quant3["quantize_frac_of_hbm"]),
                       "dequantize_frac_of_hbm": r(quant3["dequantize_frac_of_hbm"]),
                       "dequant_plus_attention_vs_bf16": r(quant3["dequant_plus_attention_ms"] / quant3["bf16_cache_attention_ms"]),
                       "fused_attention_vs_bf16": r(quant3["fused_attention_ms"] / quant3["bf16_cache_attention_ms"])}
    if others:
        l8 = others["large_8l"]
        out["large_8l"] = {"calibration_tflops": r(l8["calibration_tflops"]), "pruned_tflops": r(l8["pruned_attention_tflops"]),
                           "compaction_gbs": r(l8["compaction_gbs"]), "compaction_frac_of_hbm": r(l8["compaction_frac_of_hbm"]),
                           "compaction_kernel_frac_of_hbm": r(l8["compaction_kernel_frac_of_hbm"])}
        out["final_scale_frac_of_burst"] = {f"B{p['batch']}_{p['budget_bp']}bp": r(p["frac_of_bf16_peak"])
                                            for p in others["final_scale"]["points"]}
        out["final_scale_frac_of_sustained"] = {f"B{p['batch']}_{p['budget_bp']}bp":
                                                r(p["frac_of_sustained_bf16_peak"])
                                                for p in others["final_scale"]["points"]}
    return out


def reduce_over_ranks(x: float, op: str, world: int, device) -> float:
    """Max or sum of a host float over all ranks (timing plumbing; no data-path
    collective).  Works with NCCL (CUDA device) and gloo (CPU device)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def profile_case(case: str, reps: int):
    """Small single-kernel runs for Nsight Compute captures (inputs > L2, a
    few GB at most): 'calib' = calibration attention, 4 seeds x 16 heads at
    1024^2; 'calib16' = one calibration launch exactly as the benchmark step
    runs it (16 seeds x 16 heads, 2 GB of inputs; for single-pass DRAM
    counters); 'pruned' = pruned attention of one layer of the 32-layer
    workload (batch 8, 10% budget schedule); 'compact' = compaction of 4
    layers of that workload; 'quant' = int8 quantising compaction of those 4
    layers, then the dequantisation of each; 'quant4' / 'quant3' = 4-bit /
    3-bit quantising compaction of those 4 layers, then the dequantisation of
    each."""
    import torch
    import kv_cache_compression_cas_b200 as vark
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS[WORKLOAD]
    sides, H, D = w.sides, w.heads, w.head_dim
    S, T = len(sides), synth.n_tokens(sides)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    tau = torch.from_numpy(synth.gen_tau(1, H)).to(dev)
    bias = torch.from_numpy(synth.gen_bias(1, H, S)).to(dev)
    if case in ("calib", "calib16"):
        seeds = 4 if case == "calib" else w.n_seeds
        q, k, v = (randn_bf16((seeds, H, T, D), 10 + i, dev) for i in range(3))
        mass = torch.zeros((H, S, S), dtype=torch.float32, device=dev)
        o = torch.empty_like(q)
        for _ in range(reps):
            vark.vark_scas_accumulate(q, k, v, sides, tau, bias, mass, o, st)
    else:
        L = 1 if case == "pruned" else 4
        B = w.batch
        scas = np.random.default_rng(2).uniform(size=(L, H, S))
        keep = vark.vark_build_schedule(scas, sides, w.budget_bp, w.n_sinks)
        keep_d = torch.from_numpy(keep).to(dev)
        ho = torch.empty((L, H), dtype=torch.int32, device=dev)
        so = torch.empty((L, H, S), dtype=torch.int32, device=dev)
        pl = torch.empty((L, H, S), dtype=torch.int32, device=dev)
        lb = torch.empty(L + 1, dtype=torch.int64, device=dev)
        vark.vark_build_offsets(keep_d, sides, B, D, ho, so, pl, lb)
        k, v = (randn_bf16((L, B, H, T, D), 20 + i, dev) for i in range(2))
        total = int(lb[-1].item())
        kc = torch.empty(max(total, 8), dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        reps_c = reps if case == "compact" else 1
        if case in ("quant4", "quant3"):
            num, den = (1, 2) if case == "quant4" else (3, 8)
            quantize = vark.vark_quantize_kv_int4 if case == "quant4" else vark.vark_quantize_kv_int3
            dequantize = vark.vark_dequantize_layer_int4 if case == "quant4" else vark.vark_dequantize_layer_int3
            kq4 = torch.empty(max(num * total // den, 16), dtype=torch.uint8, device=dev)
            vq4 = torch.empty_like(kq4)
            ks4 = torch.empty((L, B, H, S, D), dtype=torch.int16, device=dev)
            vs4 = torch.empty_like(ks4)
            for _ in range(reps):
                quantize(k, v, B * H * T * D, L, B, H, sides, D, keep_d, ho, so, lb, kq4, vq4, ks4, vs4)
            base4 = lb.cpu().numpy()
            for _ in range(reps):
                for l in range(L):
                    rows = int(base4[l + 1] - base4[l]) // D
                    b0 = num * int(base4[l]) // den
                    dequantize(kq4[b0:], vq4[b0:], ks4[l], vs4[l], rows, B, H, sides, D, ho[l], so[l], kc, vc)
            reps_c = 0
        for _ in range(reps_c):
            vark.vark_compact_kv(k, v, B * H * T * D, L, B, H, sides, D, keep_d, ho, so, lb, kc, vc)
        if case == "quant":
            kq = torch.empty(max(total, 16), dtype=torch.int8, device=dev)
            vq = torch.empty_like(kq)
            ka = torch.empty((L, B, H, S, D), dtype=torch.float32, device=dev)
            va = torch.empty_like(ka)
            for _ in range(reps):
                vark.vark_quantize_kv_int8(k, v, B * H * T * D, L, B, H, sides, D, keep_d, ho, so, lb, kq, vq, ka,
                                           va)
            base = lb.cpu().numpy()
            for _ in range(reps):
                for l in range(L):
                    rows = int(base[l + 1] - base[l]) // D
                    vark.vark_dequantize_layer_int8(kq[int(base[l]):], vq[int(base[l]):], ka[l], va[l], rows, B, H,
                                                    sides, D, ho[l], so[l], kc, vc)
        if case == "pruned":
            q = randn_bf16((B, H, T, D), 30, dev)
            out = torch.empty_like(q)
            for _ in range(reps):
                vark.vark_pruned_attention(q, kc, vc, total // D, k[0], v[0], sides, -1, ho[0], so[0], pl[0], tau,
                                           bias, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    print(f"profile case {case}: ok", flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile-case", choices=["calib", "calib16", "pruned", "compact", "quant", "quant4", "quant3"],
                    default=None)
    ap.add_argument("--profile-reps", type=int, default=3)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="vark", choices=["vark", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gen-passes", type=int, default=2)
    ap.add_argument("--stability", type=int, default=1)
    ap.add_argument("--quant", type=int, default=1)
    ap.add_argument("--other-configs", type=int, default=1)
    ap.add_argument("--scas-only", type=int, default=1)
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, rank, world)
    if args.profile_case:
        return profile_case(args.profile_case, args.profile_reps)

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    max_over_ranks = lambda x: reduce_over_ranks(x, "max", world, dev)
    sum_over_ranks = lambda x: reduce_over_ranks(x, "sum", world, dev)

    w = synth.WORKLOADS[WORKLOAD]
    peaks = _peaks()
    pipe = Pipeline(w, rank, dev)
    torch.cuda.synchronize()

    for _ in range(max(args.warmup, 0)):
        pipe.step()
        assert int(pipe.status.item()) == 0, "device status after warm-up"
    torch.cuda.synchronize()

    names = ("t0", "calib", "sched", "offs", "comp", "attn")
    evs = [{k: torch.cuda.Event(enable_timing=True) for k in names} for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    pipe.launches = 0
    barrier()
    torch.cuda.synchronize()
    start.record()
    keeps = []
    for i in range(args.steps):
        keeps.append(pipe.step(evs[i]))
    stop.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    launches = pipe.launches
    assert int(pipe.status.item()) == 0, "device status after timed steps"
    elapsed = start.elapsed_time(stop) / 1e3
    t_max = max_over_ranks(elapsed)

    work = [pipe.work(k) for k in keeps]
    w_calib = sum(x["calib_flops"] for x in work)
    w_pruned = sum(x["pruned_flops"] for x in work)
    w_comp = sum(x["comp_bytes"] for x in work)
    w_qtok = sum(x["query_tokens"] for x in work)
    ph = {k: 0.0 for k in ("calib", "sched", "offs", "comp", "attn")}
    for e in evs:
        prev = "t0"
        for k in ("calib", "sched", "offs", "comp", "attn"):
            ph[k] += e[prev].elapsed_time(e[k]) / 1e3
            prev = k
    ph = {k: max_over_ranks(v) for k, v in ph.items()}
    tot_flops = sum_over_ranks(w_calib + w_pruned)
    value = tot_flops / t_max / 1e12
    K = args.steps
    L = w.layers
    calib_tflops = sum_over_ranks(w_calib) / ph["calib"] / 1e12
    pruned_tflops = sum_over_ranks(w_pruned) / ph["attn"] / 1e12
    qtok_s = sum_over_ranks(w_qtok) / ph["attn"]
    comp_gbs = sum_over_ranks(w_comp) / ph["comp"] / 1e9
    # dominant kernel: calibration attention (tensor-bound), timed inside a long step -> sustained peak
    per_launch_flops = w_calib / (K * L)
    per_launch_s = ph["calib"] / (K * L)
    traffic, traffic_note = measured_traffic()
    roof = {"bound": "tensor", "kernel": "attn_kernel<128,false,true,true> (S-CAS calibration attention, O written)",
            "achieved": per_launch_flops / per_launch_s / 1e12, "peak": peaks["bf16_tflops_sustained"],
            "unit": "TFLOP/s", "traffic": traffic, "traffic_source": "profiles/traffic.json: " + traffic_note,
            "algorithmic_bytes_per_launch": 2.0 * 4 * w.n_seeds * w.heads * pipe.T * w.head_dim,
            "peak_kind": f"bf16 dense sustained ({peaks['source']}): kernels timed inside the step"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["frac_of_burst"] = roof["achieved"] / peaks["bf16_tflops"]
    kernels = {
        "scas_calibration_attention": {"ms_per_step": ph["calib"] * 1e3 / K, "tflops": calib_tflops,
                                       "frac_of_bf16_peak": calib_tflops / peaks["bf16_tflops_sustained"]},
        "pruned_attention": {"ms_per_step": ph["attn"] * 1e3 / K, "tflops": pruned_tflops,
                             "query_tokens_per_s": qtok_s,
                             "frac_of_bf16_peak": pruned_tflops / peaks["bf16_tflops_sustained"]},
        "compaction": {"ms_per_step": ph["comp"] * 1e3 / K, "gbs": comp_gbs,
                       "frac_of_hbm_peak": comp_gbs / peaks["hbm_gbs"],
                       "bytes_per_step": w_comp / K},
        "schedule_host": {"ms_per_step": ph["sched"] * 1e3 / K},
        "offsets": {"ms_per_step": ph["offs"] * 1e3 / K},
    }

    # ------------------------------------------------ end to end through host buffers
    # Inputs come from pinned host memory every step: per-layer copies on a
    # copy stream, each layer's kernels waiting only for their own inputs;
    # outputs go back on a device-to-host stream as each layer finishes.
    e2e = None
    ke = args.e2e_steps if args.e2e_steps is not None else min(K, 3)
    if ke > 0:
        names = ("cq", "ck", "cv", "k", "v", "q")
        host_in = {name: torch.empty(getattr(pipe, name).shape, dtype=torch.bfloat16, pin_memory=True)
                   for name in names}
        for name, t in host_in.items():
            t.copy_(getattr(pipe, name))
        host_out = torch.empty(pipe.out.shape, dtype=torch.bfloat16, pin_memory=True)
        h2d = sum(t.numel() * 2 for t in host_in.values())
        d2h = host_out.numel() * 2 + pipe.mass.numel() * 4
        torch.cuda.synchronize()
        barrier()
        cs, ds = torch.cuda.Stream(), torch.cuda.Stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ework = 0.0
        for _ in range(ke):
            keep = pipe.step_streamed(host_in, host_out, cs, ds)
            x = pipe.work(keep)
            ework += x["calib_flops"] + x["pruned_flops"]
        e1.record()
        torch.cuda.synchronize()
        barrier()
        et = max_over_ranks(e0.elapsed_time(e1) / 1e3)
        e2e = {"value": sum_over_ranks(ework) / et / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": ke, "ms_per_step": et * 1e3 / ke,
               "h2d_gbs": sum_over_ranks(h2d * ke) / et / 1e9,
               "overlap": "per-layer H2D on a copy stream, D2H on a second stream, kernels wait on per-layer events"}
        del host_in, host_out

    # ------------------------------------------------ S-CAS without the attention output
    scas_o = scas_only(pipe, max_over_ranks, ph["calib"] * 1e3 / K, peaks) if args.scas_only else None

    # ------------------------------------------------ ranking stability (two disjoint seed halves)
    stab = ranking_stability(pipe) if args.stability else None

    # ------------------------------------------------ int8 retained cache
    quant = int8_cache(pipe, max_over_ranks, ph["attn"] * 1e3 / K, peaks["hbm_gbs"]) if args.quant else None
    quant4 = packed_cache(pipe, max_over_ranks, ph["attn"] * 1e3 / K, peaks["hbm_gbs"], 4) if args.quant else None
    quant3 = packed_cache(pipe, max_over_ranks, ph["attn"] * 1e3 / K, peaks["hbm_gbs"], 3) if args.quant else None

    # ------------------------------------------------ generation order (scale by scale)
    gen = None
    if args.gen_passes > 0:
        del pipe.cq, pipe.ck, pipe.cv
        torch.cuda.empty_cache()
        gen = generation_order(pipe, args.gen_passes, max_over_ranks, sum_over_ranks)

    # ------------------------------------------------ the other 1024^2 workloads (per-kernel figures)
    others = None
    if args.other_configs:
        del pipe
        torch.cuda.empty_cache()
        others = other_configs(rank, dev, max_over_ranks, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from threadpoolctl import threadpool_info
        sample = CpuSample(w)
        t0 = time.perf_counter()
        fl = 0.0
        n = 0
        while n < 1 or (time.perf_counter() - t0 < 10.0 and n < 8):
            fl += sample.run()
            n += 1
        dt = time.perf_counter() - t0
        cores = max([x.get("num_threads", 1) for x in threadpool_info()] or [1])
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": sample.describe() + f"; {n} repetitions, {dt:.1f} s", "per_step": sample.per_step()}

    # A compact copy of the per-kernel figures inside `roofline`, so that they
    # travel with the headline fields.  Convention: kernels timed inside the
    # step are set against the sustained bf16 peak, single launches timed
    # alone against the burst peak; both fractions are given for each.
    roof["per_kernel"] = summarize_kernels(kernels, quant, quant4, quant3, others, scas_o, peaks)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": t_max * 1e3 / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": arm_config(w, world),
            "pruned_attention_tflops": pruned_tflops, "query_tokens_per_s": qtok_s, "compaction_gbs": comp_gbs,
            "roofline": roof,
            # the contract's keys before the long per-section records
            "e2e": e2e, "gpu_launches": launches, "clocks": clk, "peaks": peaks, "cpu_baseline": cpu,
            "kernels": kernels, "scas_without_output": scas_o, "ranking_stability": stab,
            "int8_cache": quant, "int4_cache": quant4, "int3_cache": quant3, "generation_order": gen,
            "other_configs": others,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
