"""GPU parity of the paged-cache entry points.  A paged cache holds the same
logical entries as a contiguous one, spread over a shuffled page pool whose
unused pages are filled with NaN (any read of them would poison the result).
Each paged call must return exactly (bit for bit) what the contiguous call
returns on the gathered cache, and match the oracle; pages marked absent
(ids outside the pool) are never read or written."""
import numpy as np
import pytest
import torch

import oracle
from csa_checks import check_out, check_topk, np64

from long_context_compressed_03_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _fp8_rows(x):
    amax = x.float().abs().amax(-1)
    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    return (x.float() / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8), sc


def _page(cache, page_size, seed, extra=5, scale=None, absent_from=None):
    """Spread cache [B, N_cap, *row] over a shuffled pool of pages.  Returns a
    PagedCache; pages listed after absent_from[b] (logical page index) get the
    id -1.  Unused pool pages hold NaN (or 0xFF codes)."""
    B, N_cap = cache.shape[:2]
    row = cache.shape[2:]
    max_pages = -(-N_cap // page_size)
    num_pages = B * max_pages + extra
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages)
    if cache.dtype == torch.uint8:
        pool = torch.full((num_pages, page_size, *row), 0xFF, dtype=torch.uint8)
    else:
        pool = torch.full((num_pages, page_size, *row), float("nan"), dtype=cache.dtype)
    spool = None if scale is None else torch.full((num_pages, page_size), float("nan"))
    bt = perm.astype(np.int32)
    if absent_from is not None:
        for b, j in enumerate(absent_from):
            bt[b, j:] = -1
    for b in range(B):
        for j in range(max_pages):
            if bt[b, j] < 0:
                continue
            lo, hi = j * page_size, min(N_cap, (j + 1) * page_size)
            if lo < hi:
                pool[bt[b, j], :hi - lo] = cache[b, lo:hi]
                if scale is not None:
                    spool[bt[b, j], :hi - lo] = scale[b, lo:hi]
    return api.PagedCache(pool.to(DEV), torch.from_numpy(bt).to(DEV),
                          None if spool is None else spool.to(DEV)), max_pages * page_size


@pytest.mark.parametrize("page_size", [1, 16, 64, 256])
def test_paged_indexer_equals_contiguous_and_oracle(page_size):
    B, N_cap, H_I, d_I, k, m = 3, 5000, 4, 64, 256, 4
    g = _gen(page_size)
    qI = torch.randn(B, 1, H_I, d_I, generator=g).to(torch.bfloat16)
    codes, sc = _fp8_rows(torch.randn(B, N_cap, d_I, generator=g))
    ctx = np.array([4 * N_cap + 2, 4 * 3001 + 1, 4 * 700], np.int64)
    ne = np.minimum(ctx // m, N_cap).astype(np.int32)
    q_pos = (ctx - 1).reshape(B, 1).astype(np.int32)
    paged, cap = _page(codes, page_size, 7, scale=sc)
    kw = dict(n_entries=torch.from_numpy(ne).to(DEV), q_pos=torch.from_numpy(q_pos).to(DEV))
    idx_p = torch.empty(B, 1, k, dtype=torch.int32, device=DEV)
    api.csa_indexer_topk_paged(qI.to(DEV), paged, m, k, idx_p, **kw)
    idx_c = api.indexer_topk(qI.to(DEV), codes.to(DEV), m, k, kI_scale=sc.to(DEV), **kw)
    assert torch.equal(idx_p, idx_c)
    q_rows = oracle.quantized_query_rows(qI.float().numpy()).reshape(B, H_I, d_I)
    scores = oracle.indexer_scores_rows(q_rows, np.arange(B, dtype=np.int32), q_pos.reshape(-1),
                                        codes.numpy(), m, ne, sc.numpy())
    check_topk(idx_p.cpu().numpy().reshape(B, k), scores, k)


def test_paged_indexer_absent_pages_score_as_zero_rows():
    B, N_cap, H_I, d_I, k, m, P = 2, 3000, 4, 64, 64, 4, 64
    g = _gen(3)
    qI = torch.randn(B, 1, H_I, d_I, generator=g).to(torch.bfloat16)
    codes, sc = _fp8_rows(torch.randn(B, N_cap, d_I, generator=g))
    ne = np.array([N_cap, N_cap], np.int32)
    q_pos = np.full((B, 1), 4 * N_cap, np.int32)
    paged, _ = _page(codes, P, 11, scale=sc, absent_from=[10, 30])
    idx = torch.empty(B, 1, k, dtype=torch.int32, device=DEV)
    api.csa_indexer_topk_paged(qI.to(DEV), paged, m, k, idx,
                               n_entries=torch.from_numpy(ne).to(DEV),
                               q_pos=torch.from_numpy(q_pos).to(DEV))
    ref_codes = codes.numpy().copy()
    ref_codes[0, 10 * P:] = 0                   # absent pages read as zero rows
    ref_codes[1, 30 * P:] = 0
    q_rows = oracle.quantized_query_rows(qI.float().numpy()).reshape(B, H_I, d_I)
    scores = oracle.indexer_scores_rows(q_rows, np.arange(B, dtype=np.int32), q_pos.reshape(-1),
                                        ref_codes, m, ne, sc.numpy())
    check_topk(idx.cpu().numpy().reshape(B, k), scores, k)


def _attn_case(seed, B, H, D, N_cap, W):
    g = _gen(seed)
    q = torch.randn(B, 1, H, D, generator=g).to(torch.bfloat16)
    kv_c = torch.randn(B, N_cap, D, generator=g).to(torch.bfloat16)
    swa = torch.randn(B, W, D, generator=g).to(torch.bfloat16)
    return q, kv_c, swa


@pytest.mark.parametrize("page_size,H,D", [(16, 64, 128), (64, 16, 64), (1, 32, 128)])
def test_paged_sparse_attn_equals_contiguous_and_oracle(page_size, H, D):
    B, N_cap, W, k = 4, 3000, 256, 512
    q, kv_c, swa = _attn_case(20 + page_size, B, H, D, N_cap, W)
    ctx = np.array([12000, 9000, 700, 1], np.int64)
    ne = np.minimum(ctx // 4, N_cap)
    rng = np.random.default_rng(page_size)
    idx = np.full((B, 1, k), -1, np.int32)
    for b in range(B):
        v = int(ne[b])
        if v:
            idx[b, 0, :min(k, v)] = rng.choice(v, size=min(k, v), replace=False)
    kw = dict(raw_pos0=torch.from_numpy((ctx - W).astype(np.int32)).to(DEV),
              raw_len=torch.from_numpy(np.minimum(ctx, W).astype(np.int32)).to(DEV),
              q_pos=torch.from_numpy((ctx - 1).reshape(B, 1).astype(np.int32)).to(DEV))
    paged, _ = _page(kv_c, page_size, 5)
    qd, idd, sd = q.to(DEV), torch.from_numpy(idx).to(DEV), swa.to(DEV)
    out_p = torch.empty_like(qd)
    lse_p = torch.empty(B, 1, H, device=DEV)
    api.csa_sparse_attn_paged(qd, paged, idd, sd, W, out_p, lse_out=lse_p, **kw)
    out_c, lse_c = api.sparse_attn(qd, kv_c.to(DEV), idd, sd, W, with_lse=True, **kw)
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)
    ro, rl = oracle.sparse_attn(np64(q), np64(kv_c), idx, np64(swa), W,
                                q_pos=(ctx - 1).reshape(B, 1).astype(np.int32),
                                raw_pos0=(ctx - W).astype(np.int32),
                                raw_len=np.minimum(ctx, W).astype(np.int32))
    check_out(np64(out_p).reshape(ro.shape), ro, torch.bfloat16)


def test_paged_sparse_attn_skips_absent_pages_like_padding():
    B, H, D, N_cap, W, k, P = 2, 64, 128, 2048, 128, 256, 32
    q, kv_c, swa = _attn_case(4, B, H, D, N_cap, W)
    ctx = np.array([4 * N_cap, 4 * N_cap], np.int64)
    rng = np.random.default_rng(1)
    idx = np.stack([rng.choice(N_cap, size=k, replace=False) for _ in range(B)])[:, None].astype(np.int32)
    kw = dict(raw_pos0=torch.from_numpy((ctx - W).astype(np.int32)).to(DEV),
              raw_len=torch.full((B,), W, dtype=torch.int32, device=DEV),
              q_pos=torch.from_numpy((ctx - 1).reshape(B, 1).astype(np.int32)).to(DEV))
    paged, _ = _page(kv_c, P, 9, absent_from=[20, 50])
    out = torch.empty(B, 1, H, D, dtype=torch.bfloat16, device=DEV)
    api.csa_sparse_attn_paged(q.to(DEV), paged, torch.from_numpy(idx).to(DEV), swa.to(DEV), W, out,
                              **kw)
    ref_idx = idx.copy()
    ref_idx[0][ref_idx[0] >= 20 * P] = -1
    ref_idx[1][ref_idx[1] >= 50 * P] = -1
    ro, _ = oracle.sparse_attn(np64(q), np64(kv_c), ref_idx, np64(swa), W,
                               q_pos=(ctx - 1).reshape(B, 1).astype(np.int32),
                               raw_pos0=(ctx - W).astype(np.int32), raw_len=np.full(B, W, np.int32))
    assert not torch.isnan(out).any()
    check_out(np64(out).reshape(ro.shape), ro, torch.bfloat16)


@pytest.mark.parametrize("page_size", [8, 128])
def test_paged_hca_equals_contiguous(page_size):
    B, H, D, N_cap, W, m = 3, 64, 128, 4000, 256, 4
    q, kv_c, swa = _attn_case(30 + page_size, B, H, D, N_cap, W)
    ctx = np.array([4 * N_cap + 1, 700, 1], np.int64)
    kw = dict(n_entries=torch.from_numpy(np.minimum(ctx // m, N_cap).astype(np.int32)).to(DEV),
              raw_pos0=torch.from_numpy((ctx - W).astype(np.int32)).to(DEV),
              raw_len=torch.from_numpy(np.minimum(ctx, W).astype(np.int32)).to(DEV),
              q_pos=torch.from_numpy((ctx - 1).reshape(B, 1).astype(np.int32)).to(DEV))
    paged, _ = _page(kv_c, page_size, 2)
    qd, sd = q.to(DEV), swa.to(DEV)
    out_p = torch.empty_like(qd)
    api.hca_dense_attn_paged(qd, paged, m, sd, W, out_p, **kw)
    out_c = api.hca_attn(qd, kv_c.to(DEV), m, sd, W, **kw)
    assert torch.equal(out_p, out_c)
    ro, _ = oracle.hca_attn(np64(q), np64(kv_c), m, np64(swa), W,
                            n_entries=np.minimum(ctx // m, N_cap).astype(np.int32),
                            q_pos=(ctx - 1).reshape(B, 1).astype(np.int32),
                            raw_pos0=(ctx - W).astype(np.int32),
                            raw_len=np.minimum(ctx, W).astype(np.int32))
    check_out(np64(out_p).reshape(ro.shape), ro, torch.bfloat16)


@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_paged_compress_append_fills_the_right_pages(kind):
    B, n, d, m, P, N_cap = 3, 90, 64, 4, 4, 24
    g = _gen(8)
    x = torch.randn(B, n, d, generator=g).to(torch.bfloat16).to(DEV)
    W = (torch.randn(d, d, generator=g) / 8).to(torch.bfloat16).to(DEV)
    fp8 = kind == "e4m3"
    zero = torch.zeros(B, N_cap, d, dtype=torch.uint8 if fp8 else torch.bfloat16)
    paged, cap = _page(zero, P, 4, scale=torch.zeros(B, N_cap) if fp8 else None,
                       absent_from=[N_cap // P, N_cap // P, 3])   # element 2: pages >= 3 absent
    flat = torch.zeros(B, cap, d, dtype=zero.dtype, device=DEV)
    flat_s = torch.zeros(B, cap, device=DEV) if fp8 else None
    st_p = torch.zeros(B, 2, d, device=DEV)
    st_c = torch.zeros(B, 2, d, device=DEV)
    ne_p = torch.zeros(B, dtype=torch.int32, device=DEV)
    for p in range(n):
        pos = torch.full((B,), p, dtype=torch.int32, device=DEV)
        tok = x[:, p].contiguous()
        api.csa_compress_append_paged(tok, W, m, True, pos, st_p, paged, n_entries=ne_p)
        api.csa_compress_append(tok, W, m, True, pos, st_c, flat, cache_scale=flat_s)
    torch.cuda.synchronize()
    assert torch.equal(st_p, st_c)
    bt = paged.block_table.cpu().numpy()
    pool = paged.pool.cpu()
    written = min(n // m, cap)
    for b in range(B):
        for s in range(written):
            pg = bt[b, s // P]
            if pg < 0:
                continue
            assert torch.equal(pool[pg, s % P], flat[b, s].cpu())
            if fp8:
                assert paged.scale[pg, s % P].item() == flat_s[b, s].item()
    # absent pages were left alone: the pool's unused pages still hold their fill
    used = set(bt[bt >= 0].tolist())
    for pg in range(pool.shape[0]):
        if pg not in used:
            if fp8:
                assert torch.all(pool[pg] == 0xFF)
            else:
                assert torch.isnan(pool[pg].float()).all()
