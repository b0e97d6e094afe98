#!/usr/bin/env python
"""Benchmark of the CSA hot path on B200.

Headline: CSA prefill queries/s at n = 65536 (batch 1, 64x128 heads MQA, m = 4
overlapping, fp8 e4m3 indexer 4x64 with per-row scales, top-512, window 512,
1% 4x-norm outlier keys).  One step = the whole path over one batch:
compress(kv) -> compress(indexer keys, fp8) -> indexer + top-k -> sparse
attention.  Also reported, each with its stages' rooflines: the batch-2
n = 8192 prefill with a bf16 indexer (top-256, window 128), the HCA prefill
at n = 32768 (m' = 128, dense attention), CSA decode tok/s at 128K context
(batch 64, 32768-entry compressed cache, 512-row SWA cache, top-512; one
step = indexer + top-k -> sparse attention) and HCA decode at a 2^20-token
context.  The e4m3 tensor peak the fp8 indexer is held against is measured
here (torch._scaled_mm); the HBM and bf16 peaks come from the measured-peaks
file at the repository root.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own
batch with no collective on the data path (weak scaling); the time is the
max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_compressed_03_b200 import api, synth  # noqa: E402

PREFILL = "csa_prefill_n64k_fp8idx"
PREFILL_C2 = "csa_prefill_n8k_bf16"
HCA_PREFILL = "hca_prefill_n32k"
DECODE = "csa_decode_b64_ctx128k"
HCA_DECODE = "hca_decode_b16_ctx1m"
METRIC = "CSA prefill queries/s at n=64K & decode tok/s at 128K ctx; % HBM/TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum),
# keyed by kernel family and workload; valid only while the kernel source
# hashes the same (a changed kernel reports null traffic).
NCU_TRAFFIC = {
    # one ncu capture of the launch list at the headline workload
    ("sparse_attn", "csa_prefill_n64k_fp8idx"): {"bytes": (1231.322112 + 1024.743168) * 1e6,
                                                 "file": "attention_tc.cu", "src": "febc5b765f7c"},
    ("indexer_topk", "csa_prefill_n64k_fp8idx"): {"bytes": (39.693824 + 80.695552) * 1e6,
                                                  "file": "indexer_tc.cu", "src": "a88389db118a"},
    # the compressors' entries stay in L2 at the end of the launch (no DRAM
    # write inside it): the figure is the input read once
    ("compress_kv", "csa_prefill_n64k_fp8idx"): {"bytes": 16.852224e6, "file": "compress.cu",
                                                 "src": "5dca76459416"},
    ("compress_kI", "csa_prefill_n64k_fp8idx"): {"bytes": 8.43776e6, "file": "compress.cu",
                                                 "src": "5dca76459416"},
    # the --set full capture of the HCA prefill at its own size (n = 32768)
    ("hca_dense_attn", "hca_prefill_n32k"): {"bytes": (545.514496 + 486.443264) * 1e6,
                                             "file": "attention_tc.cu", "src": "febc5b765f7c"},
    ("compress_kv", "hca_prefill_n32k"): {"bytes": 8.461568e6, "file": "compress.cu",
                                          "src": "27570fb7979b"},
}


# ---------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def measure_fp8_peak(dev, sustain_s=1.5):
    """Dense e4m3 tensor-core throughput on this GPU: torch._scaled_mm
    (cuBLASLt) of 8192^3 e4m3 x e4m3 -> bf16 with unit per-tensor scales,
    2*N^3 flops.  Burst = best of 10 single launches (CUDA events); sustained =
    back-to-back launches for ``sustain_s`` seconds (the power cap settles
    within that)."""
    N = 8192
    g = torch.Generator(device=dev).manual_seed(7)
    a = torch.randn(N, N, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(N, N, device=dev, generator=g).to(torch.float8_e4m3fn).t()   # column-major
    one = torch.ones((), device=dev, dtype=torch.float32)
    mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(3):
        mm()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    flops = 2.0 * N ** 3
    # sustained: batches of 20 launches until sustain_s has passed; the last half counts
    times = []
    t_end = time.perf_counter() + sustain_s
    while time.perf_counter() < t_end:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(20):
            mm()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / 20)
    tail = times[len(times) // 2:] or times
    del a, b
    return {"burst": flops / (best / 1e3) / 1e12,
            "sustained": flops / (float(np.median(tail)) / 1e3) / 1e12,
            "how": "measured by bench: torch._scaled_mm e4m3 8192^3 -> bf16, best of 10 "
                   f"(burst) / median of back-to-back launches over {sustain_s} s (sustained)"}


class Peaks:
    """Roofline denominators: HBM copy GB/s and dense tensor TFLOP/s per
    operand type, burst (kernel timed alone or in a short region at full
    clock) and sustained (under the power cap)."""

    def __init__(self, peaks, src, fp8=None):
        self.hbm = peaks["hbm_gbs"]
        self.src = src
        self.tf = {("bf16", "burst"): peaks["bf16_tflops"],
                   ("bf16", "sustained"): peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])}
        # fp16 runs at the bf16 rate on the tensor cores (same nominal dense peak)
        self.tf[("f16", "burst")] = self.tf[("bf16", "burst")]
        self.tf[("f16", "sustained")] = self.tf[("bf16", "sustained")]
        if fp8:
            self.tf[("e4m3", "burst")] = fp8["burst"]
            self.tf[("e4m3", "sustained")] = fp8["sustained"]
            self.fp8_src = fp8["how"]
        else:   # the nominal dense ratio e4m3 : bf16 = 4.5 : 2.25
            self.tf[("e4m3", "burst")] = 2 * self.tf[("bf16", "burst")]
            self.tf[("e4m3", "sustained")] = 2 * self.tf[("bf16", "sustained")]
            self.fp8_src = f"2 x {src} bf16 (nominal dense ratio 4.5 : 2.25 PFLOP/s)"

    def source(self, bound, dtype, regime):
        if bound == "hbm":
            return f"{self.src} HBM copy"
        if dtype == "e4m3":
            return f"{regime} e4m3: {self.fp8_src}"
        what = "bf16 (fp16 runs at the bf16 rate)" if dtype == "f16" else "bf16"
        return f"{self.src} {regime} {what}"


def regime_of(clocks, timed_ms):
    """Burst or sustained peak for kernels timed inside a region: sustained
    when the sampled clocks show the power cap or a median SM clock more than
    7% under its maximum, or when the region is seconds long."""
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in clocks.get("reasons", [])
    low = bool(sm and smax and sm < 0.93 * smax)
    if capped or low or timed_ms > 2000.0:
        why = ("sw_power_cap active" if capped else
               f"median SM clock {sm:.0f} of {smax:.0f} MHz" if low else
               f"timed region {timed_ms / 1e3:.1f} s")
        return "sustained", why
    return "burst", (f"median SM clock {sm:.0f} of {smax:.0f} MHz, no power cap, "
                     f"timed region {timed_ms:.0f} ms" if sm else "no clock samples")


def src_hash(name: str) -> str:
    p = os.path.join(ROOT, "long_context_compressed_03_b200", "csrc", name)
    with open(p, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def ncu_traffic(key):
    tr = NCU_TRAFFIC.get(key)
    return tr["bytes"] if tr and tr["src"] == src_hash(tr["file"]) else None


def visible(t, m, ne):
    return np.minimum((t + 1) // m, ne)


def prefill_work(w):
    """Algorithmic flops / bytes per stage for one CSA prefill step: every
    input read once, every output written once (the per-unit figures of the
    design notes times the units of one launch)."""
    B, n, H, D, m, k, W = w.B, w.n, w.H, w.D, w.m, w.topk, w.window
    HI, dI = w.H_I, w.d_I
    N_c = n // m
    t = np.arange(n, dtype=np.int64)
    V = visible(t, m, N_c)
    e = 2  # bf16
    key_bytes = dI + 4 if w.indexer == "e4m3" else dI * e     # fp8 row + scale, or bf16 row
    comp_kv_bytes = B * n * D * e + B * N_c * D * e + D * D * e
    comp_kI_bytes = B * n * dI * e + B * N_c * key_bytes + dI * dI * e
    sel = V > k
    idx_flops = 2.0 * B * HI * dI * float(V[sel].sum())
    idx_bytes = B * n * HI * dI * e + B * N_c * key_bytes + B * n * k * 4
    keys = np.minimum(k, V) + np.minimum(W, t + 1)
    attn_flops = 4.0 * B * H * D * float(keys.sum())
    attn_bytes = 2 * B * n * H * D * e + B * N_c * D * e + B * n * D * e + B * n * k * 4
    return {
        "compress_kv": dict(bytes=comp_kv_bytes, flops=2.0 * B * N_c * D * D),
        "compress_kI": dict(bytes=comp_kI_bytes, flops=2.0 * B * N_c * dI * dI),
        "indexer_topk": dict(bytes=idx_bytes, flops=idx_flops),
        "sparse_attn": dict(bytes=attn_bytes, flops=attn_flops),
    }


def varlen_work(w, lens):
    """prefill_work summed over packed sequences of the given lengths (B = 1 each)."""
    tot = {}
    for L in lens:
        if L <= 0:
            continue
        for k_, v in prefill_work(dataclasses.replace(w, B=1, n=int(L))).items():
            t = tot.setdefault(k_, dict(bytes=0.0, flops=0.0))
            t["bytes"] += v["bytes"]
            t["flops"] += v["flops"]
    return tot


def hca_prefill_work(w):
    """HCA prefill: compress (m' non-overlapping) then dense attention over
    every visible entry plus the window."""
    B, n, H, D, m, W = w.B, w.n, w.H, w.D, w.m, w.window
    N_c = n // m
    t = np.arange(n, dtype=np.int64)
    keys = visible(t, m, N_c) + np.minimum(W, t + 1)
    e = 2
    return {
        "compress_kv": dict(bytes=B * n * D * e + B * N_c * D * e + D * D * e,
                            flops=2.0 * B * N_c * D * D),
        "hca_dense_attn": dict(bytes=2 * B * n * H * D * e + B * N_c * D * e + B * n * D * e,
                               flops=4.0 * B * H * D * float(keys.sum())),
    }


# Which roofline bounds each stage, and the operand type of its contraction.
STAGE_BOUND = {
    "compress_kv": ("hbm", None), "compress_kI": ("hbm", None),
    "indexer_topk": ("tensor", None),      # e4m3 or bf16, by the workload's indexer type
    "sparse_attn": ("tensor", "f16"), "hca_dense_attn": ("tensor", "f16"),
}


def roofline_of(work, ms, peaks, regime, bound=None, dtype="bf16"):
    """One kernel against its roofline: achieved flops (tensor-bound) or
    bytes (HBM-bound) per second over the peak for its operand type and
    regime.  bound=None picks by intensity against the ridge point."""
    tf = peaks.tf[(dtype, regime)]
    if bound is None:
        ridge = tf * 1e12 / (peaks.hbm * 1e9)
        bound = "tensor" if work["flops"] > ridge * max(work["bytes"], 1.0) else "hbm"
    if bound == "tensor":
        a = work["flops"] / (ms / 1e3) / 1e12
        r = {"bound": "tensor", "achieved": a, "peak": tf, "unit": "TFLOP/s", "frac": a / tf}
    else:
        a = work["bytes"] / (ms / 1e3) / 1e9
        r = {"bound": "hbm", "achieved": a, "peak": peaks.hbm, "unit": "GB/s",
             "frac": a / peaks.hbm}
    r["peak_source"] = peaks.source(r["bound"], dtype, regime)
    return r


def stage_rooflines(work, kern_ms, peaks, regime, indexer_dtype="bf16", workload=None):
    out = {}
    total = sum(kern_ms.values())
    for nm, ms in kern_ms.items():
        bound, dt = STAGE_BOUND[nm]
        if nm == "indexer_topk":
            dt = indexer_dtype
        wk = work[nm]
        out[nm] = {"ms": ms, "share": ms / max(1e-9, total),
                   "TFLOP/s": wk["flops"] / (ms / 1e3) / 1e12,
                   "GB/s": wk["bytes"] / (ms / 1e3) / 1e9,
                   "roofline": roofline_of(wk, ms, peaks, regime, bound, dt or "bf16")}
        out[nm]["roofline"]["traffic"] = ncu_traffic((nm, workload)) if workload else None
    return out


def decode_work(w, inp):
    B, H, D, k, W, HI, dI = w.B, w.H, w.D, w.topk, w.window, w.H_I, w.d_I
    ne = inp["n_entries"].numpy().astype(np.int64)
    idx_bytes = int((ne * (dI + 4)).sum()) + B * HI * dI * 2 + B * k * 4
    idx_flops = 2.0 * HI * dI * float(ne.sum())
    keys = np.minimum(k, ne) + W
    attn_bytes = int(B * k * D * 2 + B * W * D * 2 + 2 * B * H * D * 2 + B * k * 4)
    attn_flops = 4.0 * H * D * float(keys.sum())
    return {"indexer_topk": dict(bytes=idx_bytes, flops=idx_flops),
            "sparse_attn": dict(bytes=attn_bytes, flops=attn_flops)}


class ClockSampler:
    """Samples SM clock / power / throttle reasons with nvidia-smi while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        cvd = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [s.strip() for s in cvd.split(",") if s.strip()]
        self.gpu = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None
        self.lines = []
        self.error = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception as e:  # no nvidia-smi
            self.error = str(e)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        if self.error or not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": self.error or "no samples"}
        sm, smax, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "unparsed"}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------- our arm
class PrefillPath:
    """Device buffers + the four ABI calls of one CSA prefill step."""

    def __init__(self, w, inp, dev):
        self.w = w
        self.d = {k: v.to(dev) for k, v in inp.items()}
        B, n = w.B, w.n
        N_c = n // w.m
        self.fp8 = w.indexer == "e4m3"
        self.kv_c = torch.empty(B, N_c, w.D, dtype=torch.bfloat16, device=dev)
        self.kI_c = torch.empty(B, N_c, w.d_I, dtype=torch.uint8 if self.fp8 else torch.bfloat16,
                                device=dev)
        self.kI_s = torch.empty(B, N_c, dtype=torch.float32, device=dev) if self.fp8 else None
        self.idx = torch.empty(B, n, w.topk, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.d["q"])
        self.names = ["compress_kv", "compress_kI", "indexer_topk", "sparse_attn"]
        d = self.d
        self.calls = [
            lambda: api.csa_compress(d["kv"], d["W_c"], w.m, True, self.kv_c),
            lambda: api.csa_compress(d["kI_raw"], d["W_Ic"], w.m, True, self.kI_c, self.kI_s),
            lambda: api.csa_indexer_topk(d["qI"], self.kI_c, w.m, w.topk, self.idx,
                                         kI_scale=self.kI_s),
            lambda: api.csa_sparse_attn(d["q"], self.kv_c, self.idx, d["kv"], w.window,
                                        self.out),
        ]

    def step(self, record=False):
        if not record:
            for c in self.calls:
                c()
            return None
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.calls) + 1)]
        evs[0].record()
        for i, c in enumerate(self.calls):
            c()
            evs[i + 1].record()
        return evs


class HcaPrefillPath(PrefillPath):
    """The HCA prefill step: compress (m' non-overlapping) -> hca_dense_attn."""

    def __init__(self, w, inp, dev):
        self.w = w
        self.d = d = {k: v.to(dev) for k, v in inp.items()}
        self.kv_c = torch.empty(w.B, w.n // w.m, w.D, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty_like(d["q"])
        self.names = ["compress_kv", "hca_dense_attn"]
        self.calls = [
            lambda: api.csa_compress(d["kv"], d["W_c"], w.m, False, self.kv_c),
            lambda: api.hca_dense_attn(d["q"], self.kv_c, w.m, d["kv"], w.window, self.out),
        ]


def run_path(path, steps, warmup, dist_ctx):
    """Times K steps of a path bracketed by a barrier and synchronize.  The
    step time is the whole region's; a stage's time is its median over the
    steps (events between stages measure the kernel once the queue is ahead
    of the GPU, which holds after the first timed step)."""
    for _ in range(warmup):
        path.step()
    torch.cuda.synchronize()
    launches0 = api.csa_kernel_launches()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", 0)))
    per_step = []
    with clocks:
        dist_ctx.barrier()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            per_step.append(path.step(record=True))
        end.record()
        torch.cuda.synchronize()
        dist_ctx.barrier()
    launches = api.csa_kernel_launches() - launches0
    total_ms = start.elapsed_time(end)
    kern_ms = {nm: float(np.median([evs[i].elapsed_time(evs[i + 1]) for evs in per_step]))
               for i, nm in enumerate(path.names)}
    return dict(total_ms=total_ms, kern_ms=kern_ms, launches=launches, clocks=clocks.summary())


def run_variants(w, path, dev, steps, rank, peaks):
    """The NEXT-row variants of the prefill workload, each timed alone with
    CUDA events and L2 flushed between iterations (their inputs are smaller
    than L2): the gated-softmax compressor on kv, the Hadamard-rotated fp8
    compression of the indexer keys, and the indexer + top-k with gate
    weights against the rotated keys."""
    d, B, n, m = path.d, w.B, w.n, w.m
    N_c = n // m
    gw = {k: v.to(dev) for k, v in synth.gated_compressor_weights(w.D, w.D, m, True, seed=rank).items()}
    qw = synth.indexer_variant_inputs(B, n, w.H_I, seed=rank)["qI_weight"].to(dev)
    kv_g = torch.empty(B, N_c, w.D, dtype=torch.bfloat16, device=dev)
    kI_r = torch.empty(B, N_c, w.d_I, dtype=torch.uint8, device=dev)
    kI_rs = torch.empty(B, N_c, dtype=torch.float32, device=dev)
    idx = torch.empty(B, n, w.topk, dtype=torch.int32, device=dev)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    calls = {
        "compress_gated_kv": lambda: api.csa_compress_gated(d["kv"], gw["W_kv"], gw["W_gate"],
                                                            gw["ape"], m, True, kv_g),
        "compress_kI_hadamard": lambda: api.csa_compress(d["kI_raw"], d["W_Ic"], m, True, kI_r,
                                                         kI_rs, hadamard=True),
        "indexer_topk_gated_hadamard": lambda: api.csa_indexer_topk(
            d["qI"], kI_r, m, w.topk, idx, kI_scale=kI_rs, kI_rotated=True, qI_weight=qw),
    }
    e = 2
    c = 2
    work = {
        "compress_gated_kv": dict(flops=2.0 * B * n * w.D * 2 * c * w.D,
                                  bytes=B * n * w.D * e + 2 * w.D * c * w.D * e + m * c * w.D * 4
                                  + B * N_c * w.D * e),
        "compress_kI_hadamard": prefill_work(w)["compress_kI"],
        "indexer_topk_gated_hadamard": prefill_work(w)["indexer_topk"],
    }
    bounds = {"compress_gated_kv": (None, "bf16"), "compress_kI_hadamard": ("hbm", "bf16"),
              "indexer_topk_gated_hadamard": ("tensor", "e4m3")}
    out = {}
    for name, fn in calls.items():
        for _ in range(2):
            fn()
        ts = []
        for _ in range(steps):
            flush.fill_(1)
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record()
            fn()
            b_.record()
            ts.append((a_, b_))
        torch.cuda.synchronize()
        ms = float(np.median([a_.elapsed_time(b_) for a_, b_ in ts]))
        out[name] = {"ms": ms, "TFLOP/s": work[name]["flops"] / (ms / 1e3) / 1e12,
                     "GB/s": work[name]["bytes"] / (ms / 1e3) / 1e9,
                     "roofline": roofline_of(work[name], ms, peaks, "burst", *bounds[name])}
    del flush
    return out


def run_prefill_varlen(w, path, dev, steps, warmup, S=8):
    """The prefill step over S packed sequences of mixed lengths (the c3
    tokens re-cut into S documents; csa_*_varlen entry points), timed like
    the headline step (inputs larger than L2)."""
    d = path.d
    lens = synth.varlen_lengths(w.B * w.n, S, multiple=4, seed=3)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    e = api.varlen_entry_offsets(cu, w.m)
    T, E = int(cu[-1]), int(e[-1])
    q, kv = d["q"].reshape(T, w.H, w.D), d["kv"].reshape(T, w.D)
    qI, kI_raw = d["qI"].reshape(T, w.H_I, w.d_I), d["kI_raw"].reshape(T, w.d_I)
    kv_c = torch.empty(E, w.D, dtype=torch.bfloat16, device=dev)
    kI_c = torch.empty(E, w.d_I, dtype=torch.uint8, device=dev)
    kI_s = torch.empty(E, dtype=torch.float32, device=dev)
    idx = torch.empty(T, w.topk, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    names = ["compress_kv", "compress_kI", "indexer_topk", "sparse_attn"]

    def step():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        evs[0].record()
        api.csa_compress_varlen(kv, cu, d["W_c"], w.m, True, kv_c)
        evs[1].record()
        api.csa_compress_varlen(kI_raw, cu, d["W_Ic"], w.m, True, kI_c, kI_s)
        evs[2].record()
        api.csa_indexer_topk_varlen(qI, kI_c, cu, w.m, w.topk, idx, kI_scale=kI_s)
        evs[3].record()
        api.csa_sparse_attn_varlen(q, cu, kv_c, w.m, idx, kv, w.window, out)
        evs[4].record()
        return evs

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    recs = [step() for _ in range(steps)]
    torch.cuda.synchronize()
    ms = float(np.mean([r[0].elapsed_time(r[4]) for r in recs]))
    stages = {nm: float(np.median([r[i].elapsed_time(r[i + 1]) for r in recs]))
              for i, nm in enumerate(names)}
    return dict(lens=lens, T=T, ms=ms, stages=stages)


def run_e2e(w, inp, dev, steps):
    """Same step through the public API with pinned host inputs: every step
    copies its inputs host->device and reads its result (out, idx) back, and
    those copies are inside the timed region.  Steps are pipelined as a
    serving loop runs them: step i+1's inputs go up and step i-1's results
    come down while step i computes (three streams, device buffers double
    buffered, events ordering each buffer's reuse).  The serial time (copy,
    compute, copy back, one after the other) is reported beside it."""
    host = {k: v.pin_memory() for k, v in inp.items()}
    paths = [PrefillPath(w, inp, dev), PrefillPath(w, inp, dev)]
    out_host = torch.empty(paths[0].out.shape, dtype=paths[0].out.dtype).pin_memory()
    idx_host = torch.empty(paths[0].idx.shape, dtype=paths[0].idx.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size() + idx_host.numel() * idx_host.element_size()
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_comp + ev_out:
        e.record(torch.cuda.current_stream(dev))

    def issue(i):
        sl = i % 2
        p = paths[sl]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[sl])        # the step that last read these inputs is done
            for k, v in host.items():
                p.d[k].copy_(v, non_blocking=True)
            ev_in[sl].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[sl])
            s_comp.wait_event(ev_out[sl])       # this buffer's previous results were read back
            p.step()
            ev_comp[sl].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[sl])
            out_host.copy_(p.out, non_blocking=True)
            idx_host.copy_(p.idx, non_blocking=True)
            ev_out[sl].record(s_out)

    issue(0)
    issue(1)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        issue(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    end.record(s_out)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps

    # the serial form, for reference
    p = paths[0]
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        for k, v in host.items():
            p.d[k].copy_(v, non_blocking=True)
        p.step()
        out_host.copy_(p.out, non_blocking=True)
        idx_host.copy_(p.idx, non_blocking=True)
    b.record()
    torch.cuda.synchronize()
    return dict(ms=ms, serial_ms=a.elapsed_time(b) / steps, h2d=h2d, d2h=d2h)


def run_decode(dev, steps, warmup, rank):
    """One CSA decode step per batch element: the new token's compressor
    updates (kv and indexer keys, csa_compress_append), then indexer + top-k
    and sparse attention.  The decode value counts indexer + attention (the
    decode metric's definition); the append is reported as its own stage."""
    w = synth.WORKLOADS[DECODE]
    inp = synth.csa_decode_inputs(w, seed=rank)
    d = {k: v.to(dev) for k, v in inp.items()}
    idx = torch.empty(w.B, 1, w.topk, dtype=torch.int32, device=dev)
    out = torch.empty_like(d["q"])
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > L2 (126 MB)
    g = torch.Generator().manual_seed(1000 + rank)
    x_kv = torch.randn(w.B, w.D, generator=g).to(torch.bfloat16).to(dev)
    x_ki = torch.randn(w.B, w.d_I, generator=g).to(torch.bfloat16).to(dev)
    W_c = (torch.randn(w.D, w.D, generator=g) / w.D ** 0.5).to(torch.bfloat16).to(dev)
    W_Ic = (torch.randn(w.d_I, w.d_I, generator=g) / w.d_I ** 0.5).to(torch.bfloat16).to(dev)
    st_kv = torch.zeros(w.B, 2, w.D, dtype=torch.float32, device=dev)
    st_ki = torch.zeros(w.B, 2, w.d_I, dtype=torch.float32, device=dev)
    n_ent = d["n_entries"].clone()

    def step(record, split):
        """One decode step.  With split, an event between the indexer and the
        attention times each alone; without it the attention may start its
        prologue while the indexer finishes (programmatic launch), as in a
        serving loop, so the step total is timed without that event."""
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if record else None
        if record:
            evs[0].record()
        api.csa_compress_append(x_kv, W_c, w.m, True, d["q_pos"].reshape(-1), st_kv, d["kv_c"],
                                n_entries=n_ent)
        api.csa_compress_append(x_ki, W_Ic, w.m, True, d["q_pos"].reshape(-1), st_ki, d["kI_c"],
                                cache_scale=d["kI_scale"])
        if record:
            evs[1].record()
        api.csa_indexer_topk(d["qI"], d["kI_c"], w.m, w.topk, idx, kI_scale=d["kI_scale"],
                             n_entries=d["n_entries"], q_pos=d["q_pos"])
        if record and split:
            evs[2].record()
        api.csa_sparse_attn(d["q"], d["kv_c"], idx, d["swa"], w.window, out,
                            raw_pos0=d["raw_pos0"], raw_len=d["raw_len"], q_pos=d["q_pos"])
        if record:
            evs[3].record()
        return evs

    def timed(split):
        recs = []
        for _ in range(steps):
            flush.fill_(1)                     # evict the caches from L2 between steps
            recs.append(step(True, split))
        torch.cuda.synchronize()
        return recs

    for _ in range(warmup):
        step(False, False)
    torch.cuda.synchronize()
    recs = timed(False)
    t_app = [r[0].elapsed_time(r[1]) for r in recs]
    tot = [r[1].elapsed_time(r[3]) for r in recs]
    split = timed(True)
    t_idx = [r[1].elapsed_time(r[2]) for r in split]
    t_att = [r[2].elapsed_time(r[3]) for r in split]
    return dict(w=w, inp=inp, ms=float(np.mean(tot)), ms_median=float(np.median(tot)),
                kern_ms={"indexer_topk": float(np.median(t_idx)),
                         "sparse_attn": float(np.median(t_att))},
                split_ms=float(np.median([a + b for a, b in zip(t_idx, t_att)])),
                append_ms=float(np.median(t_app)))


def run_decode_paged(dev, steps, warmup, rank, page_size=64):
    """The decode step's indexer + attention over paged caches: the c4 caches
    cut into pages of page_size entries and scattered over a shuffled pool
    (serving layout), L2 flushed between steps."""
    w = synth.WORKLOADS[DECODE]
    inp = synth.csa_decode_inputs(w, seed=rank)
    d = {k: v.to(dev) for k, v in inp.items()}
    B, N_cap = d["kv_c"].shape[:2]
    max_pages = N_cap // page_size
    g = torch.Generator().manual_seed(2000 + rank)
    perm = torch.randperm(B * max_pages, generator=g).to(dev)
    bt = perm.reshape(B, max_pages).to(torch.int32).contiguous()

    def scatter(cache):
        pool = torch.empty((B * max_pages, page_size) + tuple(cache.shape[2:]), dtype=cache.dtype,
                           device=dev)
        pool[perm] = cache.reshape((B * max_pages, page_size) + tuple(cache.shape[2:]))
        return pool

    kv = api.PagedCache(scatter(d["kv_c"]), bt)
    ki = api.PagedCache(scatter(d["kI_c"]), bt, scatter(d["kI_scale"]))
    idx = torch.empty(w.B, 1, w.topk, dtype=torch.int32, device=dev)
    out = torch.empty_like(d["q"])
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        evs[0].record()
        api.csa_indexer_topk_paged(d["qI"], ki, w.m, w.topk, idx, n_entries=d["n_entries"],
                                   q_pos=d["q_pos"])
        evs[1].record()
        api.csa_sparse_attn_paged(d["q"], kv, idx, d["swa"], w.window, out,
                                  raw_pos0=d["raw_pos0"], raw_len=d["raw_len"], q_pos=d["q_pos"])
        evs[2].record()
        return evs

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    recs = []
    for _ in range(steps):
        flush.fill_(1)
        recs.append(step())
    torch.cuda.synchronize()
    t_idx = [r[0].elapsed_time(r[1]) for r in recs]
    t_att = [r[1].elapsed_time(r[2]) for r in recs]
    tot = [a + b for a, b in zip(t_idx, t_att)]
    return dict(w=w, ms=float(np.mean(tot)), page_size=page_size, work=decode_work(w, inp),
                kern_ms={"indexer_topk": float(np.median(t_idx)),
                         "sparse_attn": float(np.median(t_att))})


def run_hca_decode(dev, steps, warmup, rank):
    """HCA decode at a 2^20-token context (batch 16, 8192 entries + 512-token
    window per element): one dense attention launch per step, L2 flushed."""
    w = synth.WORKLOADS[HCA_DECODE]
    inp = synth.hca_decode_inputs(w, seed=rank)
    d = {k: v.to(dev) for k, v in inp.items()}
    out = torch.empty_like(d["q"])
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        api.hca_dense_attn(d["q"], d["kv_c"], w.m, d["swa"], w.window, out,
                           n_entries=d["n_entries"], raw_pos0=d["raw_pos0"], raw_len=d["raw_len"],
                           q_pos=d["q_pos"])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        ts.append((a, b))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ts]
    nbytes = w.B * (w.N_cap + w.window) * w.D * 2 + 2 * w.B * w.H * w.D * 2
    flops = 4.0 * w.B * w.H * w.D * (w.N_cap + w.window)
    return dict(w=w, ms=float(np.mean(ms)), ms_median=float(np.median(ms)), bytes=nbytes, flops=flops)


# ---------------------------------------------------------------------- oracle arm
def oracle_prefill_sample(w, inp, n_sample, seed=5):
    """The fp64 oracle on a bounded sample of a CSA prefill workload: both
    compressors over every token, then indexer + top-k and attention for
    n_sample sampled queries of the first sequence (fp8 indexers quantise
    keys and queries as the kernels do; bf16 ones score the bf16-stored
    keys).  Returns (seconds per query, detail)."""
    import oracle
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    B, n = w.B, w.n
    t0 = time.perf_counter()
    kv_c = oracle.compress(f64(inp["kv"]), f64(inp["W_c"]), w.m, True)
    kI_c = oracle.compress(f64(inp["kI_raw"]), f64(inp["W_Ic"]), w.m, True)
    t_comp = time.perf_counter() - t0
    rows = synth.query_sample(n, w.m, w.window, n_sample, seed=seed).numpy()[:n_sample]
    rb = np.zeros(rows.size, np.int32)
    rt = rows.astype(np.int32)
    if w.indexer == "e4m3":
        keys, scales = oracle.quantize_rows_e4m3(kI_c.astype(np.float32))
        qrows = oracle.quantized_query_rows(inp["qI"][0, rows].float().numpy())
    else:
        keys = torch.from_numpy(kI_c).to(torch.bfloat16).double().numpy()
        scales = None
        qrows = f64(inp["qI"][0, rows])
    t1 = time.perf_counter()
    idx, _, _ = oracle.indexer_topk_rows(qrows, rb, rt, keys, w.m, w.topk,
                                         np.full(B, n // w.m, np.int32), scales)
    oracle.sparse_attn_rows(f64(inp["q"][0, rows]), rb, rt, kv_c, idx, f64(inp["kv"]), w.window)
    t_rows = time.perf_counter() - t1
    per_query = t_comp / (B * n) + t_rows / rows.size
    return per_query, dict(compress_s=t_comp, rows=int(rows.size), rows_s=t_rows,
                           wall_s=time.perf_counter() - t0)


def oracle_hca_prefill_sample(w, inp, n_sample, seed=6):
    """The fp64 oracle on a bounded sample of the HCA prefill: compress every
    token, dense attention for n_sample sampled queries."""
    import oracle
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    n = w.n
    t0 = time.perf_counter()
    kv_c = oracle.compress(f64(inp["kv"]), f64(inp["W_c"]), w.m, False)
    t_comp = time.perf_counter() - t0
    rows = synth.query_sample(n, w.m, w.window, n_sample, seed=seed).numpy()[:n_sample]
    rb = np.zeros(rows.size, np.int32)
    t1 = time.perf_counter()
    oracle.hca_attn_rows(f64(inp["q"][0, rows]), rb, rows.astype(np.int32), kv_c, w.m,
                         f64(inp["kv"]), w.window)
    t_rows = time.perf_counter() - t1
    return t_comp / (w.B * n) + t_rows / rows.size, dict(compress_s=t_comp, rows=int(rows.size),
                                                         rows_s=t_rows)


def cpu_baseline(w, inp, n_sample, hca=False):
    import oracle
    fn = oracle_hca_prefill_sample if hca else oracle_prefill_sample
    per_q, det = fn(w, inp, n_sample)
    what = "the compressor" if hca else "both compressors"
    rest = "dense attention" if hca else "indexer/top-k and attention"
    return {"value": 1.0 / per_q, "unit": "queries/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"fp64 oracle: {what} over all {w.B * w.n} tokens "
                       f"({det['compress_s']:.2f} s) + {rest} for {det['rows']} of "
                       f"{w.B * w.n} queries ({det['rows_s']:.2f} s); "
                       f"queries/s = 1 / (compress_s/tokens + rows_s/rows)")}


# ---------------------------------------------------------------------- distributed
class DistCtx:
    """One process per GPU: NCCL on GPUs, gloo when run on host cores (tests).
    The data path has no collective; only the barrier around the timed region
    and the max over ranks of each timing use the process group."""

    def __init__(self, gpus=1, backend=None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.on = self.world > 1
        self.backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if self.on:
            import datetime
            import torch.distributed as dist
            kw = {}
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=300), **kw)
            self.dist = dist

    def barrier(self):
        if self.on:
            self.dist.barrier()

    def max(self, v: float) -> float:
        if not self.on:
            return v
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def job_rate(self, units_per_rank: float, ms: float) -> tuple[float, float]:
        """Whole-job throughput (units/s) of weak-scaled ranks: every rank
        processed units_per_rank in its own ms; the job takes the slowest."""
        t = self.max(ms)
        return units_per_rank * self.world / (t / 1e3), t

    def close(self):
        if self.on:
            self.dist.destroy_process_group()


CONFIGS = {
    # name: (input builder, path, HCA, oracle sample rows)
    PREFILL_C2: (synth.csa_prefill_inputs, PrefillPath, False, 8192),
    HCA_PREFILL: (synth.hca_prefill_inputs, HcaPrefillPath, True, 32768),
}


def run_config(name, dev, args, dist_ctx, rank, peaks):
    """One of the other prefill configurations, timed like the headline
    step, with its stages' rooflines and (rank 0, one GPU) the oracle's
    baseline on a sample of the same workload."""
    mk, path_cls, hca, n_cpu = CONFIGS[name]
    wc = synth.WORKLOADS[name]
    inp_c = mk(wc, seed=rank)
    pc = path_cls(wc, inp_c, dev)
    rc = run_path(pc, args.steps, args.warmup, dist_ctx)
    cval, cms = dist_ctx.job_rate(wc.B * wc.n, rc["total_ms"] / args.steps)
    creg, creg_why = regime_of(rc["clocks"], rc["total_ms"])
    cwork = hca_prefill_work(wc) if hca else prefill_work(wc)
    cst = stage_rooflines(cwork, rc["kern_ms"], peaks, creg, wc.indexer, name)
    cdom = max(rc["kern_ms"], key=rc["kern_ms"].get)
    croof = dict(cst[cdom]["roofline"], kernel=cdom, regime=f"{creg}: {creg_why}",
                 traffic=ncu_traffic((cdom, name)))
    entry = {"workload": name, "value": cval, "unit": "queries/s", "ms_per_step": cms,
             "B": wc.B, "n": wc.n, "m": wc.m, "overlap": wc.overlap,
             "l2": "inputs larger than L2 (q alone is 256 MiB or more)",
             "roofline": croof, "stages": cst, "gpu_launches": rc["launches"],
             "clocks": rc["clocks"]}
    if not hca:
        entry.update(topk=wc.topk, window=wc.window, indexer=f"{wc.indexer} {wc.H_I}x{wc.d_I}")
    else:
        entry.update(window=wc.window, attention="dense over every visible entry + window")
    if rank == 0 and dist_ctx.world == 1 and not args.no_cpu_baseline:
        entry["cpu_baseline"] = cpu_baseline(wc, inp_c, n_cpu, hca=hca)
    return entry


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-sample", type=int, default=16384,
                    help="queries the oracle baseline scores (bounded CPU sample)")
    ap.add_argument("--n", type=int, default=0,
                    help="override the prefill length (smaller cases for profiler captures; "
                         "the line is then marked as not the headline workload)")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the timing of the NEXT-row variants")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode steps (profiler captures of the decode kernels)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the c2 (n=8192, bf16 indexer) and HCA prefill (n=32768) lines")
    ap.add_argument("--only", choices=["c2", "hca"], default=None,
                    help="run only the n=8192 (c2) or the HCA n=32768 prefill (profiler "
                         "captures; the line is then not the headline)")
    ap.add_argument("--no-fp8-peak", action="store_true",
                    help="skip the e4m3 peak measurement (the nominal ratio to bf16 is used)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    w = synth.WORKLOADS[PREFILL]
    if args.n:
        w = dataclasses.replace(w, n=args.n)
    config = {"workload": PREFILL if not args.n else f"{PREFILL} (n overridden to {args.n}: "
                                                       "profiling case, not the headline)", "B": w.B, "n": w.n, "H": w.H, "D": w.D, "m": w.m,
              "overlap": True, "topk": w.topk, "window": w.window, "indexer": "e4m3 per-row scale",
              "H_I": w.H_I, "d_I": w.d_I, "outliers": "1% tokens x4", "seed": "rank",
              "l2": "inputs larger than L2 (q alone is 1 GiB); decode flushes L2 between steps",
              "parallelism": f"replicas x{args.gpus}"}

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        import oracle
        inp = synth.csa_prefill_inputs(w, seed=0)
        sample = max(16, args.cpu_sample // 16)
        for _ in range(args.warmup):
            oracle_prefill_sample(w, inp, 16)
        per_qs, walls = [], []
        for i in range(args.steps):
            per_q, det = oracle_prefill_sample(w, inp, sample, seed=10 + i)
            per_qs.append(per_q)
            walls.append(det["wall_s"])
        v = 1.0 / float(np.mean(per_qs))
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "queries/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": float(np.mean(walls)) * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded N(0,1))", "config": config,
                "cpu_baseline": {"value": v, "unit": "queries/s", "cores": oracle.num_threads(),
                                 "kind": "oracle",
                                 "sample": f"one step = both compressors over all {w.n} tokens + "
                                           f"indexer/top-k and attention for {sample} sampled "
                                           "queries (ms_per_step is that step's measured wall "
                                           "time); value = queries/s over the whole workload, "
                                           "1 / (compress_s/n + rows_s/rows)"},
                "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    dist_ctx = DistCtx(args.gpus)
    rank = dist_ctx.rank
    dev = torch.device("cuda", dist_ctx.local)
    torch.cuda.set_device(dev)
    api.load()
    raw_peaks, peak_src = load_peaks()
    if args.decode_only:
        peaks = Peaks(raw_peaks, peak_src)
        dec = run_decode(dev, args.steps, args.warmup, rank)
        hd = run_hca_decode(dev, args.steps, args.warmup, rank)
        dval, dms = dist_ctx.job_rate(dec["w"].B, dec["ms"])
        line = {"metric": "CSA decode tok/s at 128K ctx (decode only: profiling case, not the headline)",
                "value": dval, "unit": "tok/s",
                "n_gpus": dist_ctx.world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": dms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": DECODE, "hca_workload": HCA_DECODE},
                "stages_ms": dec["kern_ms"], "hca_decode_ms": dist_ctx.max(hd["ms"])}
        if rank == 0:
            print(json.dumps(line))
        dist_ctx.close()
        return 0

    if args.only:
        peaks = Peaks(raw_peaks, peak_src)
        name = PREFILL_C2 if args.only == "c2" else HCA_PREFILL
        entry = run_config(name, dev, args, dist_ctx, rank, peaks)
        line = {"metric": f"{name} prefill queries/s (profiling case, not the headline)",
                "value": entry["value"], "unit": "queries/s", "n_gpus": dist_ctx.world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": entry["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic", "config": {"workload": name},
                "detail": entry}
        if rank == 0:
            print(json.dumps(line))
        dist_ctx.close()
        return 0

    fp8 = None
    if not args.no_fp8_peak:
        try:
            fp8 = measure_fp8_peak(dev)
        except Exception as e:  # no fp8 GEMM in this torch build
            print(f"warning: fp8 peak not measured ({e})", file=sys.stderr)
    peaks = Peaks(raw_peaks, peak_src, fp8)
    torch.cuda.empty_cache()

    inp = synth.csa_prefill_inputs(w, seed=rank)
    path = PrefillPath(w, inp, dev)
    pre = run_path(path, args.steps, args.warmup, dist_ctx)
    value, ms_step = dist_ctx.job_rate(w.B * w.n, pre["total_ms"] / args.steps)
    regime, regime_why = regime_of(pre["clocks"], pre["total_ms"])
    work = prefill_work(w)
    stages = stage_rooflines(work, pre["kern_ms"], peaks, regime, "e4m3", PREFILL)
    dom = max(pre["kern_ms"], key=pre["kern_ms"].get)
    roof = {k: v for k, v in stages[dom]["roofline"].items()}
    roof["traffic"] = ncu_traffic((dom, PREFILL))
    roof["kernel"] = dom
    roof["regime"] = f"{regime}: {regime_why}"

    line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": dist_ctx.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1), 1% 4x outlier keys)", "config": config,
            "roofline": roof, "stages": stages, "gpu_launches": pre["launches"],
            "clocks": pre["clocks"],
            "peaks": {"hbm_gbs": peaks.hbm, "bf16_tflops": peaks.tf[("bf16", "burst")],
                      "bf16_tflops_sustained": peaks.tf[("bf16", "sustained")],
                      "e4m3_tflops": peaks.tf[("e4m3", "burst")],
                      "e4m3_tflops_sustained": peaks.tf[("e4m3", "sustained")],
                      "e4m3_source": peaks.fp8_src, "source": peak_src}}
    if rank == 0 and dist_ctx.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp, args.cpu_sample)

    if not args.no_configs:
        # the other two prefill configurations, each timed like the headline
        for name in (PREFILL_C2, HCA_PREFILL):
            key = "hca_prefill" if name == HCA_PREFILL else "c2_prefill"
            line[key] = run_config(name, dev, args, dist_ctx, rank, peaks)
            torch.cuda.empty_cache()

    if not args.no_variants:
        line["variants"] = {
            "workload": PREFILL, "l2": "flushed (512 MiB write) between iterations",
            "note": "NEXT rows, each timed alone: gated-softmax compressor (kv, d 128, m 4 "
                    "overlapping), Hadamard-rotated fp8 indexer keys, gated indexer + top-k "
                    "against rotated keys",
            **run_variants(w, path, dev, max(3, args.steps), rank, peaks)}
    if not args.no_variants:
        pv = run_prefill_varlen(w, path, dev, max(3, args.steps), args.warmup)
        vval, vms = dist_ctx.job_rate(pv["T"], pv["ms"])
        line["prefill_varlen"] = {
            "workload": "csa_prefill_packed8_n64k_fp8idx", "value": vval, "unit": "queries/s",
            "ms_per_step": vms, "lengths": pv["lens"], "stages_ms": pv["stages"],
            "stages": stage_rooflines(varlen_work(w, pv["lens"]), pv["stages"], peaks, regime,
                                      "e4m3"),
            "note": "the c3 tokens re-cut into 8 packed sequences (csa_*_varlen entry points); "
                    "less causal work than one 64K sequence, so not comparable to the headline"}
    if not args.no_decode:
        dec = run_decode(dev, args.steps, args.warmup, rank)
        dval, dms = dist_ctx.job_rate(dec["w"].B, dec["ms"])
        dw = decode_work(dec["w"], dec["inp"])
        dstages = {nm: {"ms": ms, "roofline": roofline_of(dw[nm], ms, peaks, "burst", "hbm")}
                   for nm, ms in dec["kern_ms"].items()}
        line["decode"] = {"workload": DECODE, "value": dval,
                          "unit": "tok/s", "ms_per_step": dms, "ms_median": dec["ms_median"],
                          "l2": "flushed (512 MiB write) between steps", "stages": dstages,
                          "compress_append_ms": dec["append_ms"],
                          "stages_sum_ms": dec["split_ms"],
                          "note": "value = batch / (indexer + attention), timed from the indexer's "
                                  "launch to the attention's end with no event between them (the "
                                  "attention starts its prologue while the indexer finishes); the "
                                  "stages come from a second loop with an event between the two "
                                  "(stages_sum_ms), and the compressor appends are timed separately"}
        dp = run_decode_paged(dev, args.steps, args.warmup, rank)
        pval, pms = dist_ctx.job_rate(dp["w"].B, dp["ms"])
        line["decode_paged"] = {"workload": DECODE, "value": pval, "unit": "tok/s",
                                "ms_per_step": pms, "page_size": dp["page_size"],
                                "stages_ms": dp["kern_ms"],
                                "roofline": {nm: roofline_of(dp["work"][nm], ms_, peaks, "burst",
                                                             "hbm")
                                             for nm, ms_ in dp["kern_ms"].items()},
                                "l2": "flushed (512 MiB write) between steps",
                                "note": "the decode step over caches scattered into a shuffled "
                                        "page pool (csa_*_paged entry points)"}
        hd = run_hca_decode(dev, args.steps, args.warmup, rank)
        hval, hms = dist_ctx.job_rate(hd["w"].B, hd["ms"])
        line["hca_decode"] = {"workload": HCA_DECODE, "value": hval,
                              "unit": "tok/s", "ms_per_step": hms, "ms_median": hd["ms_median"],
                              "l2": "flushed (512 MiB write) between steps",
                              "roofline": roofline_of(dict(bytes=hd["bytes"], flops=hd["flops"]),
                                                      hms, peaks, "burst", "hbm"),
                              "TFLOP/s": hd["flops"] / (hms / 1e3) / 1e12}
    if not args.no_e2e:
        e2e = run_e2e(w, inp, dev, max(3, args.steps // 2))
        eval_, ems = dist_ctx.job_rate(w.B * w.n, e2e["ms"])
        line["e2e"] = {"value": eval_, "unit": "queries/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": ems, "serial_ms_per_step": e2e["serial_ms"],
                       "mode": "pipelined: step i+1's h2d and step i-1's d2h overlap step i's "
                               "kernels (3 streams, double-buffered device tensors)"}
    if rank == 0:
        print(json.dumps(line))
    dist_ctx.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
