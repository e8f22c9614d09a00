#!/usr/bin/env python
"""Benchmark of the two-branch block-sparse attention forward on B200.

Workload: the 768p video-latent shape (H=24 heads, N=241920 tokens = 60 x 48 x 84, d=128,
bf16), mixture-structured Q/K with a reblock-like layout, 128-token blocks, topk_ratio 0.1.
Metric: ms per call and dense-equivalent TFLOP/s (4*H*N^2*d per call), with the roofline of
the dominant kernel (the tcgen05 attention) against the measured bf16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path: query gather + block means, anchor, key/value
gather fused with the summaries, block scoring + Top-K, two-branch attention - five kernel
launches through the C ABI on one stream, inputs resident in HBM (4.5 GB, larger than L2).
With --gpus N > 1 (launched by torchrun) every rank runs an independent replica on its own
GPU: the path has no exchange step (weak scaling, no collective on the data path).
``--impl reference`` times the float64 CPU oracle on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/call and dense-equiv TFLOP/s at 10% density, 768p shape; % tensor/HBM roofline"
UNIT = "dense-equiv TFLOP/s"
DEFAULT_WORKLOAD = "768p-24x241920-d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attention_768p_dram.json")
KERNELS = ["gather_q", "anchor", "gather_kv_summary", "route", "attend"]
KERNELS_FP8 = ["gather_q", "anchor", "gather_kv_summary", "route", "quantize", "attend"]
KERNELS_FUSED = ["gather_q", "anchor", "gather_kv_summary", "attend"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--precision", choices=["bf16", "fp8"], default="bf16",
                    help="fp8: e4m3 logit product (queries, keys, summary and context keys "
                         "quantised per group after the routing), bf16 values")
    ap.add_argument("--summaries", choices=["reweight", "meanpool"], default="reweight",
                    help="meanpool: the baseline BSA compressed branch (comparator)")
    ap.add_argument("--routing", choices=["topk", "threshold", "fused"], default="topk",
                    help="threshold: mu + tau*sigma per query block, capped at the Top-K k "
                         "(comparator); fused: the Top-K routing inside the attention kernel "
                         "(no routing launch)")
    ap.add_argument("--tau", type=float, default=1.0)
    ap.add_argument("--reblock-steps", type=int, default=5,
                    help="timed calls of the Spark-Reblock partitioner on the same Q and K, "
                         "reported under the 'reblock' key after the timed steps (0: skip)")
    ap.add_argument("--op", choices=["attention", "reblock"], default="attention",
                    help="attention: the two-branch forward (default); reblock: the "
                         "Spark-Reblock partitioner on the same workload's Q and K")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.out = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return None
        mx = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.3 * mx] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[2])
                          if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------ the hot path

class HotPath:
    """Preallocated buffers and the five step entry points of the C ABI, called with raw
    device pointers on one stream."""

    def __init__(self, x, ratio, device, fp8=False, summaries="reweight", routing="topk",
                 tau=1.0):
        from block_sparse_attention_gather_b200 import (lib, spark_bsa_workspace_layout,
                                                        workspace_views)
        self.L = lib()
        self.x = x
        Q = x["Q"]
        self.H, self.N, self.d = Q.shape
        self.nqb = x["q_offsets"].numel() - 1
        self.nkb = x["k_offsets"].numel() - 1
        self.ratio = ratio
        self.layout = spark_bsa_workspace_layout(self.H, self.N, self.d, self.nqb, self.nkb, ratio)
        self.k = self.layout.k
        # context (sink) tokens: bf16 rows are read in place, fp32 rows converted each step
        self.nc = x["Kc"].shape[1] if x.get("Kc") is not None else 0
        from block_sparse_attention_gather_b200 import spark_bsa_workspace_size_ctx
        size = spark_bsa_workspace_size_ctx(self.H, self.N, self.d, self.nqb, self.nkb, ratio,
                                            self.nc)
        self.ws = torch.empty(size, dtype=torch.uint8, device=device)
        self.convert_ctx = self.nc > 0 and Q.dtype != torch.bfloat16
        if self.convert_ctx:
            self.Kcb = torch.empty(self.H, self.nc, self.d, dtype=torch.bfloat16, device=device)
            self.Vcb = torch.empty_like(self.Kcb)
        self.v = workspace_views(self.ws, self.layout, self.H, self.N, self.d, self.nqb, self.nkb)
        self.out = torch.empty_like(Q)
        self.dtype_code = 0 if Q.dtype == torch.bfloat16 else 1
        self.stream = torch.cuda.current_stream(device)
        # FP8 logits: codes and group scales of Qp, Kp, k~ (and the context keys)
        self.fp8 = fp8
        if fp8:
            H, N, d, nqb, nkb = self.H, self.N, self.d, self.nqb, self.nkb
            u8, f32 = torch.uint8, torch.float32
            self.Qp8 = torch.empty(H, N, d, dtype=u8, device=device)
            self.Kp8 = torch.empty(H, N, d, dtype=u8, device=device)
            self.kt8 = torch.empty(H, nkb, d, dtype=u8, device=device)
            self.q_scale = torch.empty(H, nqb, dtype=f32, device=device)
            self.k_scale = torch.empty(H, nkb, dtype=f32, device=device)
            self.kt_scale = torch.empty(H, (nkb + 127) // 128, dtype=f32, device=device)
            if self.nc:
                self.Kc8 = torch.empty(H, self.nc, d, dtype=u8, device=device)
                self.kc_scale = torch.empty(H, (self.nc + 127) // 128, dtype=f32, device=device)
        self.kernels = KERNELS_FP8 if fp8 else (KERNELS_FUSED if routing == "fused" else KERNELS)
        # comparators: mean-pool summaries, threshold routing with per-row counts
        self.summaries, self.routing, self.tau = summaries, routing, tau
        if routing in ("threshold", "fused"):
            if fp8 or self.nc:
                raise SystemExit(f"{routing} routing runs without fp8 and context here")
        if routing == "fused" and not self.L.spark_bsa_fused_supported(self.d, self.nkb, float(ratio)):
            raise SystemExit("routing inside the attention kernel does not support this shape")
        if routing == "threshold":
            self.count = torch.empty(self.H, self.nqb, dtype=torch.int32, device=device)

    def _p(self, t):
        return ctypes.c_void_p(t.data_ptr())

    def step(self, events=None):
        """One pass of the whole path; if `events` (one per kernel group of self.kernels, plus
        one) is given, records one before each group and one after the last."""
        L, x, v, p = self.L, self.x, self.v, self._p
        s = ctypes.c_void_p(self.stream.cuda_stream)
        H, N, d, nqb, nkb, k = self.H, self.N, self.d, self.nqb, self.nkb, self.k
        err = p(v["err"])
        rec = (lambda i: events[i].record(self.stream)) if events else (lambda i: None)
        rec(0)
        st = L.spark_bsa_gather_q(p(x["Q"]), self.dtype_code, H, N, d, p(x["q_perm"]),
                                  p(x["q_offsets"]), nqb, p(v["Qp"]), p(v["qbar_blocks"]), err, s)
        rec(1)
        st |= L.spark_bsa_anchor(p(v["qbar_blocks"]), p(x["q_offsets"]), H, N, d, nqb,
                                 p(v["qbar"]), s)
        rec(2)
        if self.summaries == "meanpool":
            st |= L.spark_bsa_gather_kv_meanpool(p(x["K"]), p(x["V"]), self.dtype_code, H, N, d,
                                                 p(x["k_perm"]), p(x["k_offsets"]), nkb,
                                                 p(v["Kp"]), p(v["Vp"]), p(v["kbar"]),
                                                 p(v["k_tilde"]), p(v["v_tilde"]),
                                                 p(v["cbias"]), err, s)
        else:
            st |= L.spark_bsa_gather_kv_summarize(p(x["K"]), p(x["V"]), self.dtype_code, H, N,
                                                  d, p(x["k_perm"]), p(x["k_offsets"]), nkb,
                                                  p(v["qbar"]), p(v["Kp"]), p(v["Vp"]),
                                                  p(v["kbar"]), p(v["k_tilde"]), p(v["v_tilde"]),
                                                  p(v["cbias"]), err, s)
        rec(3)
        if self.routing == "fused":
            st |= L.spark_bsa_attend_fused(p(v["Qp"]), p(v["Kp"]), p(v["Vp"]), p(v["k_tilde"]),
                                           p(v["v_tilde"]), p(v["cbias"]), p(v["qbar_blocks"]),
                                           p(v["kbar"]), k, p(x["q_perm"]), p(x["q_offsets"]),
                                           nqb, p(x["k_offsets"]), nkb, H, N, d, p(self.out),
                                           self.dtype_code, p(v["sel"]), err, s)
            rec(4)
            if st != 0:
                raise RuntimeError(f"a step entry point failed (status bits {st})")
            return
        if self.routing == "threshold":
            st |= L.spark_bsa_route_threshold(p(v["qbar_blocks"]), p(v["kbar"]), H, nqb, nkb, d,
                                              float(self.tau), k, p(v["sel"]), p(self.count),
                                              err, s)
            rec(4)
            st |= L.spark_bsa_attend_var(p(v["Qp"]), p(v["Kp"]), p(v["Vp"]), p(v["k_tilde"]),
                                         p(v["v_tilde"]), p(v["cbias"]), p(v["sel"]), k,
                                         p(self.count), p(x["q_perm"]), p(x["q_offsets"]), nqb,
                                         p(x["k_offsets"]), nkb, H, N, d, p(self.out),
                                         self.dtype_code, err, s)
            rec(5)
            if st != 0:
                raise RuntimeError(f"a step entry point failed (status bits {st})")
            return
        st |= L.spark_bsa_route(p(v["qbar_blocks"]), p(v["kbar"]), H, nqb, nkb, d, k,
                                p(v["sel"]), err, s)
        rec(4)
        Kc, Vc = x.get("Kc"), x.get("Vc")
        if self.convert_ctx:
            st |= L.spark_bsa_context_bf16(p(Kc), p(Vc), self.dtype_code, H, self.nc, d,
                                           p(self.Kcb), p(self.Vcb), s)
            Kc, Vc = self.Kcb, self.Vcb
        if self.fp8:
            st |= L.spark_bsa_quantize_fp8(p(v["Qp"]), H, N, d, p(x["q_offsets"]), nqb,
                                           p(self.Qp8), p(self.q_scale), err, s)
            st |= L.spark_bsa_quantize_fp8(p(v["Kp"]), H, N, d, p(x["k_offsets"]), nkb,
                                           p(self.Kp8), p(self.k_scale), err, s)
            st |= L.spark_bsa_quantize_fp8(p(v["k_tilde"]), H, nkb, d, None, (nkb + 127) // 128,
                                           p(self.kt8), p(self.kt_scale), err, s)
            if self.nc:
                st |= L.spark_bsa_quantize_fp8(p(Kc), H, self.nc, d, None,
                                               (self.nc + 127) // 128, p(self.Kc8),
                                               p(self.kc_scale), err, s)
            rec(5)
            nc = self.nc
            st |= L.spark_bsa_attend_fp8(p(self.Qp8), p(self.q_scale), p(self.Kp8),
                                         p(self.k_scale), p(v["Vp"]), p(self.kt8),
                                         p(self.kt_scale), p(v["v_tilde"]), p(v["cbias"]),
                                         p(v["sel"]), k, p(self.Kc8) if nc else None,
                                         p(self.kc_scale) if nc else None,
                                         p(Vc) if nc else None, nc, p(x["q_perm"]),
                                         p(x["q_offsets"]), nqb, p(x["k_offsets"]), nkb, H, N,
                                         d, p(self.out), self.dtype_code, err, s)
            rec(6)
        elif self.nc == 0:
            st |= L.spark_bsa_attend(p(v["Qp"]), p(v["Kp"]), p(v["Vp"]), p(v["k_tilde"]),
                                     p(v["v_tilde"]), p(v["cbias"]), p(v["sel"]), k,
                                     p(x["q_perm"]), p(x["q_offsets"]), nqb, p(x["k_offsets"]),
                                     nkb, H, N, d, p(self.out), self.dtype_code, err, s)
            rec(5)
        else:
            st |= L.spark_bsa_attend_ctx(p(v["Qp"]), p(v["Kp"]), p(v["Vp"]), p(v["k_tilde"]),
                                         p(v["v_tilde"]), p(v["cbias"]), p(v["sel"]), k, p(Kc),
                                         p(Vc), self.nc, p(x["q_perm"]), p(x["q_offsets"]),
                                         nqb, p(x["k_offsets"]), nkb, H, N, d, p(self.out),
                                         self.dtype_code, err, s)
            rec(5)
        if st != 0:
            raise RuntimeError(f"a step entry point failed (status bits {st})")


def attention_flops(hp):
    """Algorithmic tensor-core FLOPs of one attention launch, from the selection it used:
    4 d sum_{h,A} |A| (sum_{B in S_A} |B| + nc + (nkb - k)), nc = context tokens."""
    qo = hp.x["q_offsets"].long()
    ko = hp.x["k_offsets"].long()
    qs = (qo[1:] - qo[:-1]).double()                    # [nqb]
    ks = (ko[1:] - ko[:-1]).double()                    # [nkb]
    sel = hp.v["sel"].long()                            # [H,nqb,k]
    if getattr(hp, "routing", "topk") == "threshold":   # per-row counts
        cnt = hp.count.long().to(sel.device)            # [H,nqb]
        valid = torch.arange(sel.shape[-1], device=sel.device)[None, None, :] < cnt[..., None]
        exact = (ks.to(sel.device)[sel.clamp(0, hp.nkb - 1)] * valid).sum(-1)
        cols = (exact + hp.nc + (hp.nkb - cnt)).to(qs.device)
    else:
        exact = ks[sel].sum(-1)                         # [H,nqb]
        cols = exact + hp.nc + (hp.nkb - hp.k)
    return float(4.0 * hp.d * (cols * qs[None, :]).sum().item())


def attention_issued_flops(hp):
    """Tensor-core FLOPs the attention kernel issues, padding included: every tile multiplies a
    128-row query tile (M = 128 whatever the query block's size) against its keys, over d for
    S = Q K^T and again for O += P V.  A summary tile covers 128 keys.  An exact tile (a
    selected key block or a context tile) covers 128 keys when every key block holds 128 tokens,
    else its valid rows rounded up to 16 (the kernel's variable-width tiles); so a (head, query
    block) issues 4 * 128 * d * (sum of its tiles' keys)."""
    ko = hp.x["k_offsets"].long()
    ks = (ko[1:] - ko[:-1])
    full = hp.nkb * 128 == hp.N
    width = torch.full_like(ks, 128) if full else ((ks + 15) // 16 * 16).clamp(16, 128)
    nct = -(-hp.nkb // 128)
    ctx = 0
    if hp.nc:
        rows = [min(128, hp.nc - y) for y in range(0, hp.nc, 128)]
        ctx = sum(128 if full else min(128, max(16, -(-r // 16) * 16)) for r in rows)
    sel = hp.v["sel"].long()                                 # [H,nqb,k]
    wsel = width.to(sel.device)[sel.clamp(0, hp.nkb - 1)]    # [H,nqb,k]
    if getattr(hp, "routing", "topk") == "threshold":
        cnt = hp.count.long().to(sel.device)
        valid = torch.arange(sel.shape[-1], device=sel.device)[None, None, :] < cnt[..., None]
        exact = (wsel * valid).sum(-1)
        summ = torch.where(cnt < hp.nkb, nct * 128, 0)
        keys = (exact + ctx + summ).sum().item()
    else:
        keys = wsel.sum().item() + hp.H * hp.nqb * (ctx + (nct * 128 if hp.k < hp.nkb else 0))
    return 4.0 * 128 * hp.d * float(keys)


def kernel_bytes(hp):
    """Algorithmic HBM bytes per launch of the four bandwidth-bound kernels."""
    H, N, d, nqb, nkb, k = hp.H, hp.N, hp.d, hp.nqb, hp.nkb, hp.k
    e = hp.x["Q"].element_size()
    return {
        "gather_q": H * N * d * (e + 2) + H * N * 4 + H * nqb * d * 4,
        "anchor": H * nqb * d * 4 + H * d * 4,
        "gather_kv_summary": 2 * H * N * d * (e + 2) + H * N * 4 + H * nkb * d * (4 + 2 + 2) + H * nkb * 4,
        "route": H * (nqb + nkb) * d * 4 + H * nqb * k * 4,
        # bf16 rows read once, one code byte written per value (Qp, Kp, k~, context keys)
        "quantize": (2 * H * N * d + H * nkb * d + H * hp.nc * d) * 3,
    }


def file_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# The attention kernel's compiled code depends on these sources.
ATTENTION_SOURCES = ("attention.cu", "spark_ptx.cuh", "spark_kernels.cuh", "route_step.cuh")


def attention_sources_hash():
    h = hashlib.sha256()
    for name in ATTENTION_SOURCES:
        with open(os.path.join(ROOT, "block_sparse_attention_gather_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(hp):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    try:
        with open(PROFILE_SUMMARY) as f:
            prof = json.load(f)
    except (OSError, ValueError):
        return None
    if prof.get("attention_sources_sha256_16") != attention_sources_hash():
        return None
    per_unit = prof.get("dram_bytes_per_query_block")
    if per_unit is None:
        return None
    return per_unit * hp.H * hp.nqb


# ----------------------------------------------------------------------- CPU oracle leg

def oracle_sample(w, n_heads=1, n_units=16, seed=0):
    """Times the float64 oracle on a bounded sample of workload `w`: the full summaries and
    routing of `n_heads` heads plus the attention of `n_units` query blocks; returns the
    extrapolated seconds of one full call and a description."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from block_sparse_attention_gather_b200.workloads import make_inputs
    from dataclasses import replace
    from oracle import spark_oracle as O

    ws = replace(w, H=n_heads)                 # same N, d, structure, seed; fewer heads
    x = make_inputs(ws, device="cpu")
    f64 = lambda t: t.to(torch.bfloat16).to(torch.float64).numpy()
    qo = x["q_offsets"].numpy().astype(np.int64)
    ko = x["k_offsets"].numpy().astype(np.int64)
    nqb = len(qo) - 1
    t_prep = 0.0
    t_att = 0.0
    n_att = 0
    rng = np.random.default_rng(seed)
    for h in range(n_heads):
        Q, K, V = f64(x["Q"][h]), f64(x["K"][h]), f64(x["V"][h])
        qp = x["q_perm"][h].numpy().astype(np.int64)
        kp = x["k_perm"][h].numpy().astype(np.int64)
        Kc = f64(x["Kc"][h]) if x.get("Kc") is not None else None
        Vc = f64(x["Vc"][h]) if x.get("Vc") is not None else None
        t0 = time.perf_counter()
        r = O.forward_head(Q, K, V, qp, kp, qo, ko, w.ratio, blocks=[], Kc=Kc, Vc=Vc)
        t_prep += time.perf_counter() - t0
        blocks = rng.choice(nqb, size=n_units // n_heads, replace=False)
        Qp, Kp, Vp = Q[qp], K[kp], V[kp]
        scale = 1.0 / math.sqrt(w.d)
        t0 = time.perf_counter()
        for A in blocks:
            O.attend_block(Qp[qo[A]:qo[A + 1]], Kp, Vp, ko, r.sel[A], r.k_tilde, r.v_tilde,
                           r.c, scale, Kc=Kc, Vc=Vc)
        t_att += time.perf_counter() - t0
        n_att += len(blocks)
    per_call = (t_prep / n_heads) * w.H + (t_att / n_att) * w.H * nqb
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    desc = (f"oracle (float64 numpy) on {n_heads} of {w.H} heads (summaries + routing, full) and "
            f"{n_att} of {w.H * nqb} query blocks (attention); extrapolated linearly to one "
            f"full call; measured {t_prep + t_att:.1f} s")
    return per_call, threads, desc


def dense_flops(w):
    """Dense-equivalent FLOPs of one call: every video query against every video and context
    key, 4 H N (N + nc) d."""
    return 4.0 * w.H * float(w.N) * float(w.N + w.nc) * w.d


# --------------------------------------------------------------------------------- main

def max_over_ranks(x, world, device=None):
    """The largest of every rank's value (the job's time is its slowest rank's); one
    all-reduce on the default process group when world > 1."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, work_per_step, steps, total_ms):
    """Whole-job throughput in TFLOP/s: every rank's work over the slowest rank's time."""
    return world * work_per_step * steps / (total_ms / 1e3) / 1e12


def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def run_reference(args, world, rank):
    from block_sparse_attention_gather_b200.workloads import WORKLOADS
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    times, walls = [], []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        per_call, threads, desc = oracle_sample(w, n_heads=1, n_units=4, seed=i)
        if i >= args.warmup:
            times.append(per_call)
            walls.append(time.perf_counter() - t0)
    t = statistics.mean(times)
    # each step does a bounded sample of one call's work (the share wall/t of it, by the linear
    # extrapolation), so the rate is one call's dense-equivalent work over the extrapolated
    # call time; ms_per_step is the wall time a step actually took
    value = dense_flops(w) / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
        "ms_per_call_extrapolated": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "H": w.H, "N": w.N, "d": w.d, "topk_ratio": w.ratio,
                   "block": w.block, "layout": w.layout, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


REBLOCK_METRIC = "ms/call of the Spark-Reblock partitioner (q_reuse_k), 768p shape"


def reblock_level_node_sizes(N, block):
    """(smallest, largest) node (in tokens) of every level of the partitioner's block tree: an
    m-block node gives ceil(m/2) blocks to its left child; the last block takes the remainder."""
    nb = -(-N // block)
    off = lambda b: N if b >= nb else b * block
    out, frontier = [], [(0, nb)]
    while frontier:
        sizes, nxt = [], []
        for lo, hi in frontier:
            if hi - lo >= 2:
                mid = lo + (hi - lo + 1) // 2
                sizes.append(off(hi) - off(lo))
                nxt += [(lo, mid), (mid, hi)]
        if sizes:
            out.append((min(sizes), max(sizes)))
        frontier = nxt
    return out


def reblock_level_min_nodes(N, block):
    """Smallest node (in tokens) of every level of the partitioner's block tree."""
    return [lo for lo, _ in reblock_level_node_sizes(N, block)]


def reblock_launches_per_call(N, d, block, moment_min_node=256, moment_chunk=16384):
    """Kernel launches of one partitioner call: 4 whitening kernels, the identity order and the
    offsets, and per level 11 selection/scatter kernels plus the moment kernels - one when every
    node is a single moment chunk (it runs the power iterations itself), else two - or, below
    moment_min_node tokens or at d = 64, 8 power-pass kernels."""
    n = 6
    for lo, hi in reblock_level_node_sizes(N, block):
        if d == 128 and lo >= moment_min_node:
            n += 11 + (1 if hi <= moment_chunk else 2)
        else:
            n += 11 + 8
    return n


def reblock_bytes_flops(H, N, d, block, e_in, power_iters=4, moment_min_node=256):
    """Algorithmic work of one partitioner call: the flops of the second moment and of the
    whitening (2 H N d^2 each; bf16 tensor-core MMAs for bf16 inputs), the HBM bytes of the
    whitening (read Q and K, write the bf16 unit rows), and the HBM bytes of the per-level
    passes over the unit rows with the token index: 2 passes (node moments, projection) on
    levels whose nodes hold >= moment_min_node tokens when d = 128, power_iters + 1 passes
    otherwise, plus the keys, histogram and scatter passes (4 + 4 + 4 + 8 bytes per token)."""
    flops = 2 * 2.0 * H * N * d * d
    prep_bytes = 2.0 * H * N * d * e_in + H * N * d * 2
    level_bytes = 0.0
    for m in reblock_level_min_nodes(N, block):
        passes = 2 if (d == 128 and m >= moment_min_node) else power_iters + 1
        level_bytes += H * N * (passes * (2 * d + 4) + 4 + 3 * 4 + 4 + 8)
    return flops, prep_bytes, level_bytes


def measure_reblock(Q, K, block, steps, warmup, world, device, sample_clocks=True):
    """Times the Spark-Reblock partitioner (q_reuse_k) on Q, K: `warmup` untimed calls, then
    `steps` calls bracketed by CUDA events on the launching stream (max over ranks), then the
    whitening steps alone the same way; returns a dict of the figures."""
    from block_sparse_attention_gather_b200 import (lib, spark_reblock_workspace_layout)
    H, N, d = Q.shape
    L = lib()
    lay = spark_reblock_workspace_layout(H, N, d, block)
    ws = torch.empty(lay.total, dtype=torch.uint8, device=device)
    qp = torch.empty(H, N, dtype=torch.int32, device=device)
    kp = torch.empty_like(qp)
    offs = torch.empty(lay.nb + 1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    s = ctypes.c_void_p(stream.cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    code = 0 if Q.dtype == torch.bfloat16 else 1

    def call():
        st = L.spark_reblock(p(Q), p(K), code, H, N, d, block, 0, p(qp), p(kp), p(offs), p(ws),
                             ws.numel(), s)
        if st != 0:
            raise RuntimeError(f"spark_reblock failed with status {st}")

    def prep():
        st = L.spark_reblock_whiten(p(Q), p(K), code, H, N, d, block, p(ws), ws.numel(), s)
        if st != 0:
            raise RuntimeError(f"spark_reblock_whiten failed with status {st}")

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    clocks = ClockSampler(device) if sample_clocks else None
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(steps):
        call()
    ev[1].record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop() if clocks else None
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[1]), world, device)
    ms = total_ms / steps
    pe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    pe[0].record(stream)
    for _ in range(steps):
        prep()
    pe[1].record(stream)
    torch.cuda.synchronize()
    prep_ms = max_over_ranks(pe[0].elapsed_time(pe[1]), world, device) / steps
    part_ms = ms - prep_ms
    flops, prep_bytes, level_bytes = reblock_bytes_flops(H, N, d, block, Q.element_size())
    del ws, qp, kp, offs
    return {"ms": ms, "prep_ms": prep_ms, "levels_ms": part_ms, "flops": flops,
            "prep_bytes": prep_bytes, "level_bytes": level_bytes, "levels": lay.levels,
            "clocks": clock_info,
            "launches_per_call": reblock_launches_per_call(N, d, block)}


def run_reblock(args, world, rank, local):
    from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = WORKLOADS[args.workload]
    x = make_inputs(w, device=device)
    Q, K = x["Q"], x["K"]
    del x
    H, N, d = Q.shape
    block = w.block
    peaks, peak_kind = load_peaks()
    r = measure_reblock(Q, K, block, args.steps, args.warmup, world, device)
    ms, prep_ms, part_ms = r["ms"], r["prep_ms"], r["levels_ms"]
    flops, prep_bytes, level_bytes = r["flops"], r["prep_bytes"], r["level_bytes"]
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gbs = level_bytes / (part_ms / 1e3) / 1e9
    line = {
        "impl": "ours", "op": "reblock", "metric": REBLOCK_METRIC, "value": ms, "unit": "ms",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if Q.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": w.name, "H": H, "N": N, "d": d, "block": block,
                   "levels": r["levels"], "mode": "q_reuse_k", "power_iters": 4,
                   "l2": "inputs larger than L2, no flush"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "traffic": None,
                     "kernel": "per-level passes (power, project, select, scatter)",
                     "algorithmic_bytes_per_call": level_bytes},
        "kernels": {"whiten (second moment, M^1/2, unit rows)": {
                        "ms": prep_ms, "TFLOP/s": flops / (prep_ms / 1e3) / 1e12,
                        "flops": flops, "bytes": prep_bytes,
                        "GB/s": prep_bytes / (prep_ms / 1e3) / 1e9,
                        "units": ("tcgen05 bf16 MMAs, fp32 accumulation" if
                                  Q.dtype == torch.bfloat16 and d == 128 else "fp32 CUDA cores")},
                    "levels": {"ms": part_ms, "GB/s": gbs, "bytes": level_bytes}},
        "gpu_launches": r["launches_per_call"] * args.steps,
        "clocks": r["clocks"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        # the CPU oracle needs no process group and no GPU: rank 0 times it, the other ranks of
        # a multi-rank launch exit at once
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    world, rank, local = init_dist()
    if args.op == "reblock" and args.impl == "ours":
        run_reblock(args, world, rank, local)
        return
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps are required")
    from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = WORKLOADS[args.workload]
    x = make_inputs(w, device=device)
    hp = HotPath(x, w.ratio, device, fp8=args.precision == "fp8", summaries=args.summaries,
                 routing=args.routing, tau=args.tau)
    if hp.fp8 and hp.d != 128:
        raise SystemExit("--precision fp8 needs d = 128")
    peaks, peak_kind = load_peaks()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        hp.step()
    torch.cuda.synchronize()
    flags = int(hp.v["err"].item())
    if flags:
        raise RuntimeError(f"device error word {flags:#x} after warm-up")

    names = hp.kernels
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
           for _ in range(args.steps)]
    clocks = ClockSampler(device)
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        hp.step(evs[i])
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()

    per_kernel = {n: [] for n in names}
    totals = []
    for e in evs:
        for j, n in enumerate(names):
            per_kernel[n].append(e[j].elapsed_time(e[j + 1]))
        totals.append(e[0].elapsed_time(e[len(names)]))
    total_ms = max_over_ranks(sum(totals), world, device)
    ms_per_step = total_ms / args.steps
    dflops = dense_flops(w)
    value = whole_job_rate(world, dflops, args.steps, total_ms)
    flags = int(hp.v["err"].item())
    if flags:
        raise RuntimeError(f"device error word {flags:#x} after the timed region")

    att_flops = attention_flops(hp)
    issued_flops = attention_issued_flops(hp)
    att_ms = statistics.mean(per_kernel["attend"])
    achieved = att_flops / (att_ms / 1e3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_note = f"bf16 sustained, {peak_kind}"
    if hp.fp8:
        # half of the FLOPs (Q K^T) run at the fp8 rate, twice bf16's (nominal 4.5 / 2.25
        # PFLOP/s), half (P V) at bf16's: the mix's peak is 4/3 of bf16's
        peak = peak * 4.0 / 3.0
        peak_note = (f"bf16 sustained ({peak_kind}) x 4/3: Q K^T at fp8 = 2x bf16 (nominal "
                     "ratio), P V at bf16")
    kb = kernel_bytes(hp)
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    kernels = {}
    for n in names:
        ms = statistics.mean(per_kernel[n])
        entry = {"ms": ms, "share": ms / ms_per_step}
        if n in kb:
            gbs = kb[n] / (ms / 1e3) / 1e9
            entry.update({"bytes": kb[n], "GB/s": gbs, "hbm_frac": gbs / hbm_peak})
        else:
            issued = issued_flops / (ms / 1e3) / 1e12
            entry.update({"flops": att_flops, "TFLOP/s": achieved, "tensor_frac": achieved / peak,
                          "issued_flops": issued_flops, "issued_TFLOP/s": issued,
                          "issued_tensor_frac": issued / peak,
                          "valid_share_of_issued": att_flops / issued_flops})
        kernels[n] = entry

    # ---- end to end through the public call with host buffers (pinned), copies timed
    e2e = None
    comparator = args.summaries != "reweight" or args.routing != "topk"
    if args.e2e_steps > 0 and not comparator:      # the public calls run the method itself
        from block_sparse_attention_gather_b200 import (spark_bsa_forward_host,
                                                        spark_bsa_host_staging_size_ex,
                                                        spark_bsa_workspace_size_ctx,
                                                        spark_bsa_workspace_size_fp8)
        names = ["Q", "K", "V", "q_perm", "k_perm", "q_offsets", "k_offsets"]
        if hp.nc:
            names += ["Kc", "Vc"]
        host = {n: x[n].to("cpu").pin_memory() for n in names}
        out_host = torch.empty(hp.out.shape, dtype=hp.out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = out_host.numel() * out_host.element_size()
        s = torch.cuda.current_stream(device)
        # the host-buffer entry point, pipelined head by head (every variant: context rows and
        # FP8 logits included)
        hpc = 1
        staging = torch.empty(spark_bsa_host_staging_size_ex(hp.H, hp.N, hp.d, hp.out.dtype,
                                                             hp.nqb, hp.nkb, hpc, hp.nc),
                              dtype=torch.uint8, device=device)
        ws_size = (spark_bsa_workspace_size_fp8(1, hp.N, hp.d, hp.nqb, hp.nkb, w.ratio, hp.nc)
                   if hp.fp8 else
                   spark_bsa_workspace_size_ctx(1, hp.N, hp.d, hp.nqb, hp.nkb, w.ratio, hp.nc))
        chunk_ws = torch.empty(ws_size, dtype=torch.uint8, device=device)
        pipe = (s, torch.cuda.Stream(device), torch.cuda.Stream(device))

        def e2e_step():
            spark_bsa_forward_host(host["Q"], host["K"], host["V"], host["q_perm"],
                                   host["k_perm"], host["q_offsets"], host["k_offsets"],
                                   w.ratio, out=out_host, heads_per_chunk=hpc,
                                   staging=staging, workspace=chunk_ws, streams=pipe,
                                   Kc=host.get("Kc"), Vc=host.get("Vc"), fp8=hp.fp8)

        e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(s)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(s)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        e2e = {"value": whole_job_rate(world, dflops, args.e2e_steps, e_ms), "unit": UNIT,
               "ms_per_call": e_ms / args.e2e_steps, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "call": (f"spark_bsa_forward_host{' (FP8 logits)' if hp.fp8 else ''}"
                        f"{' with context rows' if hp.nc else ''} (host buffers, chunks of "
                        f"{hpc} heads, copies overlapped with computation on three streams)")}
        del host, out_host, staging, chunk_ws

    # ---- the partitioner upstream of the path, on the same Q and K (its own timed calls)
    reblock = None
    if args.reblock_steps > 0 and not comparator and not hp.fp8 and not hp.nc:
        r = measure_reblock(x["Q"], x["K"], w.block, args.reblock_steps, 2, world, device,
                            sample_clocks=False)
        gbs = r["level_bytes"] / (r["levels_ms"] / 1e3) / 1e9
        reblock = {"ms_per_call": r["ms"], "whiten_ms": r["prep_ms"],
                   "levels_ms": r["levels_ms"], "levels_GB/s": gbs,
                   "levels_hbm_frac": gbs / hbm_peak, "levels_bytes": r["level_bytes"],
                   "steps": args.reblock_steps, "mode": "q_reuse_k", "block": w.block,
                   "note": "separate timed calls after the timed steps; not part of value"}

    traffic = profiled_traffic(hp)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3 logits, bf16 values" if hp.fp8 else "bf16", "data": "synthetic",
        "config": {"workload": w.name, "H": w.H, "N": w.N, "d": w.d, "topk_ratio": w.ratio,
                   "k": hp.k, "nqb": hp.nqb, "nkb": hp.nkb, "context_tokens": hp.nc,
                   "block": w.block, "summaries": args.summaries, "routing": args.routing,
                   **({"tau": args.tau} if args.routing == "threshold" else {}),
                   "layout": w.layout, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (4.5 GB of Q/K/V per call), no flush"},
        "actual_tflops": att_flops / (ms_per_step / 1e3) / 1e12 * world,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_kind": peak_note,
                     "kernel": "attend (tcgen05 two-branch attention)",
                     "algorithmic_flops_per_launch": att_flops,
                     "frac_of_burst": achieved / peaks.get("bf16_tflops",
                                                           FALLBACK_PEAKS["bf16_tflops"]) *
                                      (0.75 if hp.fp8 else 1.0)},
        "kernels": kernels,
        "gpu_launches": ((4 if args.routing == "fused" else 5) + (2 if hp.convert_ctx else 0) +
                         ((4 if hp.nc else 3) if hp.fp8 else 0)) * args.steps,
        "clocks": clock_info,
        "e2e": e2e,
        "reblock": reblock,
    }
    # the CPU leg times the bf16 oracle: it is reported for the bf16 line only
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not hp.fp8 and not comparator:
        per_call, threads, desc = oracle_sample(w, n_heads=2, n_units=320)
        line["cpu_baseline"] = {"value": dflops / per_call / 1e12, "unit": UNIT,
                                "cores": threads, "kind": "oracle", "sample": desc,
                                "ms_per_call_extrapolated": per_call * 1e3}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
