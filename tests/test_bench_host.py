"""Host-side arithmetic of bench.py: the algorithmic work model and the
roofline position it reports, checked against direct counts on small
workloads (no GPU)."""
import dataclasses
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_compressed_03_b200 import synth  # noqa: E402

RAW = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
PEAKS = bench.Peaks(RAW, "measured")


def _small():
    return dataclasses.replace(synth.WORKLOADS["csa_prefill_n64k_fp8idx"], n=96, topk=5, window=7)


def test_attention_flops_count_every_key_of_every_query():
    w = _small()
    keys = 0
    for t in range(w.n):
        V = min((t + 1) // w.m, w.n // w.m)
        keys += min(w.topk, V) + min(w.window, t + 1)
    assert bench.prefill_work(w)["sparse_attn"]["flops"] == 4.0 * w.H * w.D * keys


def test_indexer_flops_count_scored_rows_only():
    w = _small()
    scored = sum(min((t + 1) // w.m, w.n // w.m) for t in range(w.n)
                 if min((t + 1) // w.m, w.n // w.m) > w.topk)
    assert bench.prefill_work(w)["indexer_topk"]["flops"] == 2.0 * w.H_I * w.d_I * scored


def test_packed_work_is_the_sum_of_its_sequences():
    w = _small()
    lens = [40, 0, 56]
    tot = bench.varlen_work(w, lens)
    a = bench.prefill_work(dataclasses.replace(w, n=40))
    b = bench.prefill_work(dataclasses.replace(w, n=56))
    for k in tot:
        assert tot[k]["flops"] == a[k]["flops"] + b[k]["flops"]
        assert tot[k]["bytes"] == a[k]["bytes"] + b[k]["bytes"]


def test_roofline_picks_the_bound_by_intensity():
    ridge = 1600e12 / 6000e9                       # flops per byte at the burst peak
    hot = bench.roofline_of({"flops": 2 * ridge * 1e6, "bytes": 1e6}, 1.0, PEAKS, "burst")
    assert hot["bound"] == "tensor" and hot["unit"] == "TFLOP/s"
    assert hot["frac"] == pytest.approx(2 * ridge * 1e6 / 1e-3 / 1e12 / 1600.0)
    cold = bench.roofline_of({"flops": 1e6, "bytes": 1e9}, 2.0, PEAKS, "sustained")
    assert cold["bound"] == "hbm" and cold["achieved"] == pytest.approx(500.0)
    assert cold["frac"] == pytest.approx(500.0 / 6000.0)
    # under the power cap the sustained tensor figure is the peak
    assert bench.roofline_of({"flops": 1e15, "bytes": 1.0}, 1.0, PEAKS, "sustained")["peak"] == 1400.0


def test_stage_bounds_and_operand_peaks():
    # fp8 indexer against the e4m3 peak, attention (fp16 operands) at the bf16 rate
    pk = bench.Peaks(RAW, "measured", {"burst": 3000.0, "sustained": 2600.0, "how": "test"})
    work = {"indexer_topk": {"flops": 3e12, "bytes": 1e6}, "sparse_attn": {"flops": 1.6e12, "bytes": 1e6},
            "compress_kv": {"flops": 1e12, "bytes": 6e9}}
    st = bench.stage_rooflines(work, {"indexer_topk": 2.0, "sparse_attn": 2.0, "compress_kv": 2.0},
                               pk, "burst", "e4m3")
    assert st["indexer_topk"]["roofline"]["peak"] == 3000.0
    assert st["indexer_topk"]["roofline"]["frac"] == pytest.approx(1500.0 / 3000.0)
    assert st["sparse_attn"]["roofline"]["peak"] == 1600.0
    # compress is HBM-bound whatever its flop count
    assert st["compress_kv"]["roofline"]["bound"] == "hbm"
    assert st["compress_kv"]["roofline"]["achieved"] == pytest.approx(3000.0)
    assert sum(s["share"] for s in st.values()) == pytest.approx(1.0)
    # no fp8 measurement: the nominal 2x of bf16, said so
    nom = bench.Peaks(RAW, "measured")
    assert nom.tf[("e4m3", "sustained")] == 2800.0 and "nominal" in nom.fp8_src


def test_regime_follows_the_sampled_clocks():
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.regime_of(full, 90.0)[0] == "burst"
    assert bench.regime_of(dict(full, reasons=["sw_power_cap"]), 90.0)[0] == "sustained"
    assert bench.regime_of(dict(full, sm_mhz=1500.0), 90.0)[0] == "sustained"
    assert bench.regime_of(full, 4000.0)[0] == "sustained"


def test_hca_prefill_work_counts_visible_entries_and_window():
    w = dataclasses.replace(synth.WORKLOADS["hca_prefill_n32k"], n=1000, window=37)
    keys = sum(min((t + 1) // w.m, w.n // w.m) + min(w.window, t + 1) for t in range(w.n))
    assert bench.hca_prefill_work(w)["hca_dense_attn"]["flops"] == 4.0 * w.H * w.D * keys


def test_varlen_lengths_are_block_aligned_and_sum_to_the_total():
    lens = synth.varlen_lengths(65536, 8, multiple=4, seed=3)
    assert sum(lens) == 65536 and len(lens) == 8
    assert all(L % 4 == 0 and L > 0 for L in lens)
    assert np.std(lens) > 0
