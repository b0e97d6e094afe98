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

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


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
    hot = bench.roofline_of({"flops": 2 * ridge * 1e6, "bytes": 1e6}, 1.0, PEAKS, True)
    assert hot["bound"] == "tensor" and hot["unit"] == "TFLOP/s"
    assert hot["frac"] == pytest.approx(2 * ridge * 1e6 / 1e-3 / 1e12 / 1600.0)
    cold = bench.roofline_of({"flops": 1e6, "bytes": 1e9}, 2.0, PEAKS, False)
    assert cold["bound"] == "hbm" and cold["achieved"] == pytest.approx(500.0)
    assert cold["frac"] == pytest.approx(500.0 / 6000.0)
    # inside a long step the sustained tensor figure is the peak
    assert bench.roofline_of({"flops": 1e15, "bytes": 1.0}, 1.0, PEAKS, False)["peak"] == 1400.0


def test_varlen_lengths_are_block_aligned_and_sum_to_the_total():
    lens = synth.varlen_lengths(65536, 8, multiple=4, seed=3)
    assert sum(lens) == 65536 and len(lens) == 8
    assert all(L % 4 == 0 and L > 0 for L in lens)
    assert np.std(lens) > 0
