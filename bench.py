#!/usr/bin/env python
"""Benchmark of the CSA hot path on B200.

Headline: CSA prefill queries/s at n = 65536 (batch 1, 64x128 heads MQA, m = 4
overlapping, fp8 e4m3 indexer 4x64 with per-row scales, top-512, window 512,
1% 4x-norm outlier keys).  One step = the whole path over one batch:
compress(kv) -> compress(indexer keys, fp8) -> indexer + top-k -> sparse
attention.  Also reported: CSA decode tok/s at 128K context (batch 64,
32768-entry compressed cache, 512-row SWA cache, top-512; one step =
indexer + top-k -> sparse attention).

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
DECODE = "csa_decode_b64_ctx128k"
HCA_DECODE = "hca_decode_b16_ctx1m"
METRIC = "CSA prefill queries/s at n=64K & decode tok/s at 128K ctx; % HBM/TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum),
# keyed by kernel family; valid only while the kernel source hashes the same.
NCU_TRAFFIC = {
    # the ncu capture of the prefill attention at n=16384: 307.4 MB read + 220.4 MB
    # written, scaled by 4 (units = queries) to one n=65536 launch
    "sparse_attn": {"bytes": (307.403008e6 + 220.389120e6) * 4, "file": "attention_tc.cu",
                    "src": "ee13d0b93b5e"},
}


# ---------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_hash(name: str) -> str:
    p = os.path.join(ROOT, "long_context_compressed_03_b200", "csrc", name)
    with open(p, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def visible(t, m, ne):
    return np.minimum((t + 1) // m, ne)


def prefill_work(w):
    """Algorithmic flops / bytes per stage for one prefill step (see DESIGN)."""
    B, n, H, D, m, k, W = w.B, w.n, w.H, w.D, w.m, w.topk, w.window
    HI, dI = w.H_I, w.d_I
    N_c = n // m
    t = np.arange(n, dtype=np.int64)
    V = visible(t, m, N_c)
    e = 2  # bf16
    comp_kv_bytes = B * n * D * e + B * N_c * D * e + D * D * e
    comp_kI_bytes = B * n * dI * e + B * N_c * (dI * 1 + 4) + dI * dI * e
    sel = V > k
    idx_flops = 2.0 * B * HI * dI * float(V[sel].sum())
    idx_bytes = B * n * HI * dI * e + B * N_c * (dI + 4) + B * n * k * 4
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


def roofline_of(work, ms, peaks, timed_alone):
    """Where one kernel sits against the roofline its algorithmic intensity
    picks (ridge = measured bf16 TFLOP/s over measured HBM GB/s): achieved
    flops or bytes per second over that peak.  Kernels timed alone use the
    burst bf16 figure, kernels inside a long step the sustained one."""
    tf = peaks["bf16_tflops"] if timed_alone else peaks.get("bf16_tflops_sustained",
                                                              peaks["bf16_tflops"])
    ridge = tf * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if work["flops"] > ridge * max(work["bytes"], 1.0):
        a = work["flops"] / (ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": a, "peak": tf, "unit": "TFLOP/s", "frac": a / tf}
    a = work["bytes"] / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": a / peaks["hbm_gbs"]}


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
    """Device buffers + the four ABI calls of one prefill step."""

    def __init__(self, w, inp, dev):
        self.w = w
        self.d = {k: v.to(dev) for k, v in inp.items()}
        B, n = w.B, w.n
        N_c = n // w.m
        self.kv_c = torch.empty(B, N_c, w.D, dtype=torch.bfloat16, device=dev)
        self.kI_c = torch.empty(B, N_c, w.d_I, dtype=torch.uint8, device=dev)
        self.kI_s = torch.empty(B, N_c, dtype=torch.float32, device=dev)
        self.idx = torch.empty(B, n, w.topk, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.d["q"])
        self.names = ["compress_kv", "compress_kI", "indexer_topk", "sparse_attn"]
        self.ev = None

    def step(self, record=False):
        d, w = self.d, self.w
        calls = [
            lambda: api.csa_compress(d["kv"], d["W_c"], w.m, True, self.kv_c),
            lambda: api.csa_compress(d["kI_raw"], d["W_Ic"], w.m, True, self.kI_c, self.kI_s),
            lambda: api.csa_indexer_topk(d["qI"], self.kI_c, w.m, w.topk, self.idx,
                                         kI_scale=self.kI_s),
            lambda: api.csa_sparse_attn(d["q"], self.kv_c, self.idx, d["kv"], w.window,
                                        self.out),
        ]
        if not record:
            for c in calls:
                c()
            return None
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
        evs[0].record()
        for i, c in enumerate(calls):
            c()
            evs[i + 1].record()
        return evs


def run_prefill(w, dev, steps, warmup, dist_ctx, rank):
    inp = synth.csa_prefill_inputs(w, seed=rank)
    path = PrefillPath(w, inp, dev)
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
    kern_ms = {nm: 0.0 for nm in path.names}
    for evs in per_step:
        for i, nm in enumerate(path.names):
            kern_ms[nm] += evs[i].elapsed_time(evs[i + 1])
    kern_ms = {k: v / steps for k, v in kern_ms.items()}
    return dict(total_ms=total_ms, kern_ms=kern_ms, launches=launches, clocks=clocks.summary(),
                path=path, inp=inp)


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
        ms = float(np.mean([a_.elapsed_time(b_) for a_, b_ in ts]))
        out[name] = {"ms": ms, "TFLOP/s": work[name]["flops"] / (ms / 1e3) / 1e12,
                     "GB/s": work[name]["bytes"] / (ms / 1e3) / 1e9,
                     "roofline": roofline_of(work[name], ms, peaks, timed_alone=True)}
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
    stages = {nm: float(np.mean([r[i].elapsed_time(r[i + 1]) for r in recs]))
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

    def step(record):
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
        if record:
            evs[2].record()
        api.csa_sparse_attn(d["q"], d["kv_c"], idx, d["swa"], w.window, out,
                            raw_pos0=d["raw_pos0"], raw_len=d["raw_len"], q_pos=d["q_pos"])
        if record:
            evs[3].record()
        return evs

    for _ in range(warmup):
        step(False)
    torch.cuda.synchronize()
    recs = []
    for _ in range(steps):
        flush.fill_(1)                     # evict the caches from L2 between steps
        recs.append(step(True))
    torch.cuda.synchronize()
    t_app = [r[0].elapsed_time(r[1]) for r in recs]
    t_idx = [r[1].elapsed_time(r[2]) for r in recs]
    t_att = [r[2].elapsed_time(r[3]) for r in recs]
    tot = [a + b for a, b in zip(t_idx, t_att)]
    return dict(w=w, inp=inp, ms=float(np.mean(tot)), ms_median=float(np.median(tot)),
                kern_ms={"indexer_topk": float(np.mean(t_idx)), "sparse_attn": float(np.mean(t_att))},
                append_ms=float(np.mean(t_app)))


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
                kern_ms={"indexer_topk": float(np.mean(t_idx)), "sparse_attn": float(np.mean(t_att))})


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
    """The fp64 oracle on a bounded sample of the prefill workload: both
    compressors over the whole sequence, then indexer + top-k and attention
    for n_sample sampled queries.  Returns (seconds per query, detail)."""
    import oracle
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    n = w.n
    t0 = time.perf_counter()
    kv_c = oracle.compress(f64(inp["kv"]), f64(inp["W_c"]), w.m, True)
    kI_c = oracle.compress(f64(inp["kI_raw"]), f64(inp["W_Ic"]), w.m, True)
    t_comp = time.perf_counter() - t0
    codes, scales = oracle.quantize_rows_e4m3(kI_c.astype(np.float32))
    rows = synth.query_sample(n, w.m, w.window, n_sample, seed=seed).numpy()[:n_sample]
    rb = np.zeros(rows.size, np.int32)
    rt = rows.astype(np.int32)
    qrows = oracle.quantized_query_rows(inp["qI"][0, rows].float().numpy())
    t1 = time.perf_counter()
    idx, _, _ = oracle.indexer_topk_rows(qrows, rb, rt, codes, w.m, w.topk,
                                         np.array([n // w.m], np.int32), scales)
    oracle.sparse_attn_rows(f64(inp["q"][0, rows]), rb, rt, kv_c, idx, f64(inp["kv"]), w.window)
    t_rows = time.perf_counter() - t1
    per_query = t_comp / n + t_rows / rows.size
    return per_query, dict(compress_s=t_comp, rows=int(rows.size), rows_s=t_rows)


def cpu_baseline(w, inp, n_sample):
    import oracle
    per_q, det = oracle_prefill_sample(w, inp, n_sample)
    return {"value": 1.0 / per_q, "unit": "queries/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"fp64 oracle: both compressors over all {w.n} tokens "
                       f"({det['compress_s']:.2f} s) + indexer/top-k and attention for "
                       f"{det['rows']} of {w.n} queries ({det['rows_s']:.2f} s); "
                       f"queries/s = 1 / (compress_s/n + rows_s/rows)")}


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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-sample", type=int, default=4096,
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
        sample = max(16, args.cpu_sample // 4)
        times = []
        for _ in range(args.warmup):
            oracle_prefill_sample(w, inp, 16)
        for i in range(args.steps):
            per_q, det = oracle_prefill_sample(w, inp, sample, seed=10 + i)
            times.append(per_q)
        per_q = float(np.mean(times))
        v = 1.0 / per_q
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "queries/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": per_q * w.n * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))",
                "config": config,
                "cpu_baseline": {"value": v, "unit": "queries/s", "cores": oracle.num_threads(),
                                 "kind": "oracle",
                                 "sample": f"{sample} sampled queries per step + full compress, "
                                           f"extrapolated to n={w.n}"},
                "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    dist_ctx = DistCtx(args.gpus)
    rank = dist_ctx.rank
    dev = torch.device("cuda", dist_ctx.local)
    torch.cuda.set_device(dev)
    api.load()
    peaks, peak_src = load_peaks()
    if args.decode_only:
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

    pre = run_prefill(w, dev, args.steps, args.warmup, dist_ctx, rank)
    value, ms_step = dist_ctx.job_rate(w.B * w.n, pre["total_ms"] / args.steps)

    work = prefill_work(w)
    dom = max(pre["kern_ms"], key=pre["kern_ms"].get)
    dom_work = work[dom]
    tensor_kernels = {"sparse_attn", "indexer_topk"}
    if dom in tensor_kernels:
        achieved = dom_work["flops"] / (pre["kern_ms"][dom] / 1e3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak}
    else:
        achieved = dom_work["bytes"] / (pre["kern_ms"][dom] / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak}
    tr = NCU_TRAFFIC.get(dom)
    roof["traffic"] = tr["bytes"] if tr and tr["src"] == src_hash(tr["file"]) else None
    roof["kernel"] = dom
    roof["peak_source"] = f"{peak_src} ({'sustained bf16' if roof['unit'] == 'TFLOP/s' else 'hbm copy'})"
    stages = {}
    for nm, ms in pre["kern_ms"].items():
        wk = work[nm]
        stages[nm] = {"ms": ms, "share": ms / max(1e-9, sum(pre["kern_ms"].values())),
                      "TFLOP/s": wk["flops"] / (ms / 1e3) / 1e12,
                      "GB/s": wk["bytes"] / (ms / 1e3) / 1e9}

    line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": dist_ctx.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1), 1% 4x outlier keys)", "config": config,
            "roofline": roof, "stages": stages, "gpu_launches": pre["launches"],
            "clocks": pre["clocks"]}

    if not args.no_variants:
        line["variants"] = {
            "workload": PREFILL, "l2": "flushed (512 MiB write) between iterations",
            "note": "NEXT rows, each timed alone: gated-softmax compressor (kv, d 128, m 4 "
                    "overlapping), Hadamard-rotated fp8 indexer keys, gated indexer + top-k "
                    "against rotated keys",
            **run_variants(w, pre["path"], dev, max(3, args.steps), rank, peaks)}
    if not args.no_variants:
        pv = run_prefill_varlen(w, pre["path"], dev, max(3, args.steps), args.warmup)
        vval, vms = dist_ctx.job_rate(pv["T"], pv["ms"])
        line["prefill_varlen"] = {
            "workload": "csa_prefill_packed8_n64k_fp8idx", "value": vval, "unit": "queries/s",
            "ms_per_step": vms, "lengths": pv["lens"], "stages_ms": pv["stages"],
            "roofline": {nm: roofline_of(wk, pv["stages"][nm], peaks, timed_alone=False)
                         for nm, wk in varlen_work(w, pv["lens"]).items()},
            "note": "the c3 tokens re-cut into 8 packed sequences (csa_*_varlen entry points); "
                    "less causal work than one 64K sequence, so not comparable to the headline"}
    if not args.no_decode:
        dec = run_decode(dev, args.steps, args.warmup, rank)
        dval, dms = dist_ctx.job_rate(dec["w"].B, dec["ms"])
        dw = decode_work(dec["w"], dec["inp"])
        dstages = {nm: {"ms": ms, "GB/s": dw[nm]["bytes"] / (ms / 1e3) / 1e9,
                        "frac_hbm": dw[nm]["bytes"] / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
                   for nm, ms in dec["kern_ms"].items()}
        line["decode"] = {"workload": DECODE, "value": dval,
                          "unit": "tok/s", "ms_per_step": dms, "ms_median": dec["ms_median"],
                          "l2": "flushed (512 MiB write) between steps", "stages": dstages,
                          "compress_append_ms": dec["append_ms"],
                          "note": "value = batch / (indexer + attention); the two compressor "
                                  "appends of the step are timed separately"}
        dp = run_decode_paged(dev, args.steps, args.warmup, rank)
        pval, pms = dist_ctx.job_rate(dp["w"].B, dp["ms"])
        line["decode_paged"] = {"workload": DECODE, "value": pval, "unit": "tok/s",
                                "ms_per_step": pms, "page_size": dp["page_size"],
                                "stages_ms": dp["kern_ms"],
                                "roofline": {nm: roofline_of(dp["work"][nm], ms_, peaks, True)
                                             for nm, ms_ in dp["kern_ms"].items()},
                                "l2": "flushed (512 MiB write) between steps",
                                "note": "the decode step over caches scattered into a shuffled "
                                        "page pool (csa_*_paged entry points)"}
        hd = run_hca_decode(dev, args.steps, args.warmup, rank)
        hval, hms = dist_ctx.job_rate(hd["w"].B, hd["ms"])
        line["hca_decode"] = {"workload": HCA_DECODE, "value": hval,
                              "unit": "tok/s", "ms_per_step": hms, "ms_median": hd["ms_median"],
                              "l2": "flushed (512 MiB write) between steps",
                              "GB/s": hd["bytes"] / (hms / 1e3) / 1e9,
                              "frac_hbm": hd["bytes"] / (hms / 1e3) / 1e9 / peaks["hbm_gbs"],
                              "TFLOP/s": hd["flops"] / (hms / 1e3) / 1e12}
    if not args.no_e2e:
        e2e = run_e2e(w, pre["inp"], dev, max(3, args.steps // 2))
        eval_, ems = dist_ctx.job_rate(w.B * w.n, e2e["ms"])
        line["e2e"] = {"value": eval_, "unit": "queries/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": ems, "serial_ms_per_step": e2e["serial_ms"],
                       "mode": "pipelined: step i+1's h2d and step i-1's d2h overlap step i's "
                               "kernels (3 streams, double-buffered device tensors)"}
    if rank == 0 and dist_ctx.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, pre["inp"], args.cpu_sample)
    if rank == 0:
        print(json.dumps(line))
    dist_ctx.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
