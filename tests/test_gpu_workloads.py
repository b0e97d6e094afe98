"""GPU parity on the five workloads at their full sizes, in the launch
configuration the benchmark times, checked stage by stage against the fp64
oracle: compression on every entry, top-k on sampled query rows (oracle fed
the GPU's own stored fp8 keys, so both sides rank the same quantised values),
attention on sampled rows (oracle fed the GPU's index rows, so a near-tie
swap cannot fail a tolerance), plus the fully independent oracle pipeline on
the fp32 workload."""
import numpy as np
import pytest
import torch

import oracle
from csa_checks import (ATOL_BF16, ATOL_F32, check_compress_stored, check_e4m3_rows, check_out,
                        check_topk, compress_bound, max_abs, np64, record)
from long_context_compressed_03_b200 import api, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _take(t, rows, shape):
    """fp64 copy of the listed rows of t viewed as `shape` (rows gathered first)."""
    idx = torch.as_tensor(np.asarray(rows), dtype=torch.long, device=t.device)
    return np64(t.reshape(shape).index_select(0, idx))


def _dev(d):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _prefill_run(w, inp):
    d = _dev(inp)
    res = api.csa_prefill(d["q"], d["kv"], d["qI"], d["kI_raw"], d["W_c"], d["W_Ic"], w.m,
                          w.topk, w.window, indexer_fp8=(w.indexer == "e4m3"))
    torch.cuda.synchronize()
    return d, res


def _check_prefill(w, inp, d, res, rows, atol):
    B, n = inp["kv"].shape[:2]
    # stage 1: both compressors, every entry
    kv_c_ref = oracle.compress(np64(inp["kv"]), np64(inp["W_c"]), w.m, True)
    kv_b = compress_bound(np64(inp["kv"]), np64(inp["W_c"]), w.m, True)
    check_compress_stored(np64(res["kv_c"]), kv_c_ref, kv_b, res["kv_c"].dtype, label="compress kv")
    kI_ref = oracle.compress(np64(inp["kI_raw"]), np64(inp["W_Ic"]), w.m, True)
    kI_b = compress_bound(np64(inp["kI_raw"]), np64(inp["W_Ic"]), w.m, True)
    if res["kI_scale"] is not None:
        codes = res["kI_c"].cpu().numpy()
        scale = res["kI_scale"].cpu().numpy()
        check_e4m3_rows(codes, scale, kI_ref, kI_b, label="compress fp8 indexer keys")
        kI_for_oracle, kI_scale = codes, scale
    else:
        check_compress_stored(np64(res["kI_c"]), kI_ref, kI_b, res["kI_c"].dtype,
                              label="compress indexer keys")
        kI_for_oracle, kI_scale = np64(res["kI_c"]), None
    # stage 2: top-k on sampled rows, the oracle scoring the GPU's stored keys
    rows = np.asarray(rows, np.int64)
    rb = (rows // n).astype(np.int32)
    rt = (rows % n).astype(np.int32)
    qrows = _take(inp["qI"], rows, (B * n, w.H_I, w.d_I))
    if kI_scale is not None:
        qrows = oracle.quantized_query_rows(qrows.astype(np.float32))
    ne = np.full(B, n // w.m, np.int32)
    scores = oracle.indexer_scores_rows(qrows, rb, rt, kI_for_oracle, w.m, ne, kI_scale)
    gidx = res["idx"].cpu().numpy().reshape(B * n, w.topk)[rows]
    stats = check_topk(gidx, scores, w.topk)
    print(f"top-k rows checked: {stats}")
    # stage 3: attention on the same rows with the GPU's index rows
    q_rows = _take(inp["q"], rows, (B * n, w.H, w.D))
    ro, _ = oracle.sparse_attn_rows(q_rows, rb, rt, np64(res["kv_c"]), gidx, np64(inp["kv"]),
                                    w.window)
    got = _take(res["out"], rows, (B * n, w.H, w.D))
    check_out(got, ro, res["out"].dtype)
    return stats


def test_csa_prefill_n512_fp32_full_and_independent_pipeline():
    w = synth.WORKLOADS["csa_prefill_n512_f32"]
    inp = synth.csa_prefill_inputs(w, seed=0)
    d, res = _prefill_run(w, inp)
    rows = np.arange(w.B * w.n)
    _check_prefill(w, inp, d, res, rows, ATOL_F32)
    # the oracle's own pipeline, sharing nothing with the GPU's intermediates
    o, _, idx = oracle.csa_forward(np64(inp["q"]), np64(inp["kv"]), np64(inp["qI"]),
                                   np64(inp["kI_raw"]), np64(inp["W_c"]), np64(inp["W_Ic"]),
                                   w.m, w.topk, w.window)
    gidx = res["idx"].cpu().numpy().reshape(-1, w.topk)
    same = np.array([np.array_equal(np.sort(a), np.sort(b)) for a, b in zip(gidx, idx)])
    # every row, matching or not, against the oracle pipeline's own scores:
    # a row whose set differs from the oracle's must be a near-tie
    n = w.n
    rows = np.arange(w.B * n)
    kI_ref = oracle.compress(np64(inp["kI_raw"]), np64(inp["W_Ic"]), w.m, True)
    scores = oracle.indexer_scores_rows(np64(inp["qI"]).reshape(-1, w.H_I, w.d_I),
                                        (rows // n).astype(np.int32), (rows % n).astype(np.int32),
                                        kI_ref, w.m, np.full(w.B, n // w.m, np.int32))
    stats = check_topk(gidx, scores, w.topk, label="c1 top-k vs the oracle pipeline")
    assert stats["exact"] + stats["near_ties"] == rows.size
    record("c1 rows whose set differs from the oracle pipeline", rows=int((~same).sum()))
    got = np64(res["out"]).reshape(-1, w.H, w.D)
    check_out(got[same], o[same], torch.float32, label="c1 outputs vs the oracle pipeline")


def test_csa_prefill_n8k_bf16():
    w = synth.WORKLOADS["csa_prefill_n8k_bf16"]
    inp = synth.csa_prefill_inputs(w, seed=0)
    d, res = _prefill_run(w, inp)
    qs = synth.query_sample(w.n, w.m, w.window, 256, seed=2).numpy()
    rows = np.concatenate([qs, w.n + qs])
    _check_prefill(w, inp, d, res, rows, ATOL_BF16)
    # run-to-run determinism of the whole path
    _, res2 = _prefill_run(w, inp)
    assert torch.equal(res["idx"], res2["idx"]) and torch.equal(res["out"], res2["out"])


def test_csa_prefill_n64k_fp8_indexer():
    w = synth.WORKLOADS["csa_prefill_n64k_fp8idx"]
    inp = synth.csa_prefill_inputs(w, seed=0)
    d, res = _prefill_run(w, inp)
    rows = synth.query_sample(w.n, w.m, w.window, 384, seed=3).numpy()
    _check_prefill(w, inp, d, res, rows, ATOL_BF16)


def test_csa_decode_b64_ctx128k():
    w = synth.WORKLOADS["csa_decode_b64_ctx128k"]
    inp = synth.csa_decode_inputs(w, seed=0)
    d = _dev(inp)
    idx = api.indexer_topk(d["qI"], d["kI_c"], w.m, w.topk, kI_scale=d["kI_scale"],
                           n_entries=d["n_entries"], q_pos=d["q_pos"])
    out = api.sparse_attn(d["q"], d["kv_c"], idx, d["swa"], w.window, raw_pos0=d["raw_pos0"],
                          raw_len=d["raw_len"], q_pos=d["q_pos"])
    torch.cuda.synchronize()
    sel = np.arange(0, w.B, 8)                      # 8 of the 64 elements
    ne = inp["n_entries"].numpy()[sel]
    qp = inp["q_pos"].numpy()[sel, 0]
    qrows = oracle.quantized_query_rows(np64(inp["qI"])[sel, 0].astype(np.float32))
    rb = np.arange(sel.size, dtype=np.int32)
    codes = inp["kI_c"].numpy()[sel]
    scales = inp["kI_scale"].numpy()[sel]
    scores = oracle.indexer_scores_rows(qrows, rb, qp, codes, w.m, ne, scales)
    gidx = idx.cpu().numpy()[sel, 0]
    check_topk(gidx, scores, w.topk)
    ro, _ = oracle.sparse_attn_rows(np64(inp["q"])[sel, 0], rb, qp, np64(inp["kv_c"][sel]), gidx,
                                    np64(inp["swa"][sel]), w.window,
                                    raw_pos0=inp["raw_pos0"].numpy()[sel],
                                    raw_len=inp["raw_len"].numpy()[sel])
    check_out(np64(out)[sel, 0], ro, out.dtype)


def test_hca_decode_b16_ctx1m():
    w = synth.WORKLOADS["hca_decode_b16_ctx1m"]
    inp = synth.hca_decode_inputs(w, seed=0)
    d = _dev(inp)
    out = api.hca_attn(d["q"], d["kv_c"], w.m, d["swa"], w.window, n_entries=d["n_entries"],
                       raw_pos0=d["raw_pos0"], raw_len=d["raw_len"], q_pos=d["q_pos"])
    torch.cuda.synchronize()
    rb = np.arange(w.B, dtype=np.int32)
    ro, _ = oracle.hca_attn_rows(np64(inp["q"])[:, 0], rb, inp["q_pos"].numpy()[:, 0],
                                 np64(inp["kv_c"]), w.m, np64(inp["swa"]), w.window,
                                 n_entries=inp["n_entries"].numpy(),
                                 raw_pos0=inp["raw_pos0"].numpy(), raw_len=inp["raw_len"].numpy())
    check_out(np64(out)[:, 0], ro, out.dtype)


def test_hca_prefill_n32k():
    w = synth.WORKLOADS["hca_prefill_n32k"]
    inp = synth.hca_prefill_inputs(w, seed=0)
    d = _dev(inp)
    kv_c = api.compress(d["kv"], d["W_c"], w.m, False)
    out = api.hca_attn(d["q"], kv_c, w.m, d["kv"], w.window)
    torch.cuda.synchronize()
    ref_c = oracle.compress(np64(inp["kv"]), np64(inp["W_c"]), w.m, False)
    check_compress_stored(np64(kv_c), ref_c, compress_bound(np64(inp["kv"]), np64(inp["W_c"]), w.m, False),
                          kv_c.dtype, label="HCA compress m'=128")
    rows = synth.query_sample(w.n, w.m, w.window, 256, seed=4).numpy()
    rows = np.unique(np.concatenate([rows, np.arange(126, 131), np.arange(w.n - 3, w.n)]))
    rb = np.zeros(rows.size, np.int32)
    ro, _ = oracle.hca_attn_rows(_take(inp["q"], rows, (w.n, w.H, w.D)), rb,
                                 rows.astype(np.int32), np64(kv_c), w.m, np64(inp["kv"]), w.window)
    check_out(_take(out, rows, (w.n, w.H, w.D)), ro, out.dtype)
