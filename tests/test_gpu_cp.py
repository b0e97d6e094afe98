"""The context-parallel prefill on one GPU (one rank, no exchange) with this
library's kernels as the arithmetic: the positioned (decode-shaped) kernels
serve a shard's queries, and the result must match the oracle."""
import numpy as np
import pytest
import torch

import oracle
from csa_checks import check_out, check_topk, np64

from long_context_compressed_03_b200 import cp

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_single_rank_cp_prefill_matches_oracle():
    n, H, D, H_I, d_I, m, k, W = 1024, 64, 128, 4, 64, 4, 64, 128
    g = torch.Generator().manual_seed(6)
    bf = lambda *s, std=1.0: (torch.randn(*s, generator=g) * std).to(torch.bfloat16)
    q, kv, qI, kI_raw = bf(n, H, D), bf(n, D), bf(n, H_I, d_I), bf(n, d_I)
    W_c, W_Ic = bf(D, D, std=D ** -0.5), bf(d_I, d_I, std=d_I ** -0.5)
    sh = cp.shard_of(n, 1, 0, m)
    res = cp.cp_prefill(sh, q.to(DEV), kv.to(DEV), qI.to(DEV), kI_raw.to(DEV), W_c.to(DEV),
                        W_Ic.to(DEV), m, k, W, cp.CudaBackend())
    torch.cuda.synchronize()
    ref_kv = oracle.compress(np64(kv)[None], np64(W_c), m, True)
    check_out(np64(res["kv_c"])[None], ref_kv, torch.bfloat16)
    codes, scales = res["kI_c"].cpu().numpy()[None], res["kI_scale"].cpu().numpy()[None]
    q_rows = oracle.quantized_query_rows(qI.float().numpy())
    t = np.arange(n, dtype=np.int32)
    scores = oracle.indexer_scores_rows(q_rows, np.zeros(n, np.int32), t, codes, m,
                                        np.array([n // m], np.int32), scales)
    idx = res["idx"].cpu().numpy()
    check_topk(idx, scores, k)
    ro, _ = oracle.sparse_attn(np64(q)[None], np64(res["kv_c"])[None], idx[None], np64(kv)[None], W)
    check_out(np64(res["out"])[None], ro, torch.bfloat16)
