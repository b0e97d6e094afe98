"""Seeded synthetic inputs for the CSA / HCA workloads.

This module is the one piece shared by the CUDA path's tests/benchmark and
the fp64 oracle: it draws the input tensors and nothing else.  It holds none
of the method's arithmetic (no pooling, projection of compressed entries,
scoring, selection or attention); the only arithmetic here builds INPUTS:
the hidden-state projections of the small fp32 workload (model layers that
sit outside the compressed-attention path) and the per-row fp8 encoding of a
decode-time indexer cache, done with torch's own float8 cast.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)``
in fp32, in the order each builder documents, then cast to the workload's
dtype.  Tensors are batch-first and contiguous:

* q      [B, n_q, H, D]      query heads (MQA: one shared KV head)
* kv     [B, n, D]           raw KV rows (key = value, shared-KV)
* qI     [B, n_q, H_I, d_I]  indexer query heads
* kI_raw [B, n, d_I]         raw indexer key rows
* W_c    [D, D], W_Ic [d_I, d_I]   compression projections, stored [in, out]
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape/precision description of one workload (no tensors)."""
    name: str
    kind: str                  # "csa_prefill" | "csa_decode" | "hca_decode" | "hca_prefill"
    B: int
    n: int                     # tokens (prefill) or max context (decode)
    H: int
    D: int
    m: int
    overlap: bool
    window: int
    H_I: int = 0
    d_I: int = 0
    topk: int = 0
    dtype: str = "bf16"        # "f32" | "bf16" (attention / KV dtype)
    indexer: str = "bf16"      # "f32" | "bf16" | "e4m3"
    outlier_frac: float = 0.0
    N_cap: int = 0             # decode caches: entries held per batch element
    ctx_lo: int = 0            # decode: context length range (inclusive)
    ctx_hi: int = 0
    hidden: int = 0            # fp32 workload: hidden size of x

    @property
    def n_entries(self) -> int:
        return self.n // self.m


WORKLOADS = {
    # CSA prefill, 1 sequence, n=512, fp32 (hidden 128, 8x64 query heads,
    # d_kv 64, m=4 overlapping, indexer 1x32, top-8, window 32).
    "csa_prefill_n512_f32": Workload("csa_prefill_n512_f32", "csa_prefill", B=1, n=512, H=8, D=64,
                                     m=4, overlap=True, window=32, H_I=1, d_I=32, topk=8,
                                     dtype="f32", indexer="f32", hidden=128),
    # CSA prefill, batch 2, n=8192, bf16, 64x128 heads, indexer 4x64 bf16, top-256, window 128.
    "csa_prefill_n8k_bf16": Workload("csa_prefill_n8k_bf16", "csa_prefill", B=2, n=8192, H=64,
                                     D=128, m=4, overlap=True, window=128, H_I=4, d_I=64,
                                     topk=256, dtype="bf16", indexer="bf16"),
    # CSA prefill, batch 1, n=65536, bf16, indexer 4x64 fp8 e4m3 per-row scale,
    # top-512, window 512, 1% of tokens with 4x-norm outlier keys.
    "csa_prefill_n64k_fp8idx": Workload("csa_prefill_n64k_fp8idx", "csa_prefill", B=1, n=65536,
                                        H=64, D=128, m=4, overlap=True, window=512, H_I=4,
                                        d_I=64, topk=512, dtype="bf16", indexer="e4m3",
                                        outlier_frac=0.01),
    # CSA decode, batch 64, 128K context as a 32768-entry compressed cache +
    # 512-row SWA cache, indexer 4x64 fp8, top-512; context ~ U[65536, 131072].
    "csa_decode_b64_ctx128k": Workload("csa_decode_b64_ctx128k", "csa_decode", B=64, n=131072,
                                       H=64, D=128, m=4, overlap=True, window=512, H_I=4, d_I=64,
                                       topk=512, dtype="bf16", indexer="e4m3", N_cap=32768,
                                       ctx_lo=65536, ctx_hi=131072),
    # HCA decode, batch 16, m'=128 over a 2^20-token context (8192 entries) + 512 SWA.
    "hca_decode_b16_ctx1m": Workload("hca_decode_b16_ctx1m", "hca_decode", B=16, n=1 << 20, H=64,
                                     D=128, m=128, overlap=False, window=512, dtype="bf16",
                                     N_cap=8192, ctx_lo=1 << 20, ctx_hi=1 << 20),
    # HCA prefill, n=32768, m'=128 non-overlapping, window 512.
    "hca_prefill_n32k": Workload("hca_prefill_n32k", "hca_prefill", B=1, n=32768, H=64, D=128,
                                 m=128, overlap=False, window=512, dtype="bf16"),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _randn(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def _encode_rows_e4m3(rows: torch.Tensor):
    """fp8 cache rows as inputs: per-row scale amax/448 and torch's E4M3 cast."""
    amax = rows.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (rows / scale.unsqueeze(-1)).to(torch.float8_e4m3fn)
    return codes.view(torch.uint8), scale.to(torch.float32)


def csa_prefill_inputs(w: Workload, seed: int = 0, n: int | None = None, B: int | None = None):
    """Inputs of a CSA prefill (positions 0..n-1 of each sequence).

    Draw order (fp32, N(0,1) unless stated): q, kv, qI, kI_raw,
    W_c ~ N(0, 1/D), W_Ic ~ N(0, 1/d_I), then the outlier positions
    (``randperm(n)`` per batch element, first floor(frac*n) taken) whose kv and
    kI_raw rows are multiplied by 4.  ``n``/``B`` override the workload's
    sizes (smaller parity cases with the same recipe).

    The fp32 workload instead draws x ~ N(0,1) [B, n, hidden] and the
    projections W_q [hidden, H*D], W_kv [hidden, D], W_c [D, D],
    W_Iq [hidden, H_I*d_I], W_Ik [hidden, d_I], W_Ic [d_I, d_I] ~ N(0, 1/fan_in)
    in that order; q, kv, qI and kI_raw are x times those projections
    (computed in fp64, stored in fp32)."""
    n = w.n if n is None else n
    B = w.B if B is None else B
    g = torch.Generator().manual_seed(seed)
    H, D, H_I, d_I = w.H, w.D, w.H_I, w.d_I
    if w.hidden:
        hid = w.hidden
        x = _randn(g, (B, n, hid))
        W_q = _randn(g, (hid, H * D), 1.0 / math.sqrt(hid))
        W_kv = _randn(g, (hid, D), 1.0 / math.sqrt(hid))
        W_c = _randn(g, (D, D), 1.0 / math.sqrt(D))
        W_Iq = _randn(g, (hid, H_I * d_I), 1.0 / math.sqrt(hid))
        W_Ik = _randn(g, (hid, d_I), 1.0 / math.sqrt(hid))
        W_Ic = _randn(g, (d_I, d_I), 1.0 / math.sqrt(d_I))
        xd = x.double()
        q = (xd @ W_q.double()).float().reshape(B, n, H, D)
        kv = (xd @ W_kv.double()).float()
        qI = (xd @ W_Iq.double()).float().reshape(B, n, H_I, d_I)
        kI_raw = (xd @ W_Ik.double()).float()
        return dict(q=q.contiguous(), kv=kv.contiguous(), qI=qI.contiguous(),
                    kI_raw=kI_raw.contiguous(), W_c=W_c, W_Ic=W_Ic)
    q = _randn(g, (B, n, H, D))
    kv = _randn(g, (B, n, D))
    qI = _randn(g, (B, n, H_I, d_I))
    kI_raw = _randn(g, (B, n, d_I))
    W_c = _randn(g, (D, D), 1.0 / math.sqrt(D))
    W_Ic = _randn(g, (d_I, d_I), 1.0 / math.sqrt(d_I))
    n_out = int(math.floor(w.outlier_frac * n))
    if n_out:
        for b in range(B):
            pos = torch.randperm(n, generator=g)[:n_out]
            kv[b, pos] *= 4.0
            kI_raw[b, pos] *= 4.0
    dt = torch_dtype(w.dtype)
    idt = torch.float32 if w.indexer == "f32" else torch.bfloat16
    return dict(q=q.to(dt), kv=kv.to(dt), qI=qI.to(idt), kI_raw=kI_raw.to(idt), W_c=W_c.to(dt),
                W_Ic=W_Ic.to(idt))


def csa_decode_inputs(w: Workload, seed: int = 0, B: int | None = None, N_cap: int | None = None,
                      ctx_lo: int | None = None, ctx_hi: int | None = None):
    """Inputs of one CSA decode step: one new query per batch element.

    Draw order: q [B,1,H,D], kv_c cache [B,N_cap,D], qI [B,1,H_I,d_I],
    kI cache rows [B,N_cap,d_I] (N(0,1), then per-row fp8 with scale
    amax/448), SWA cache [B,W,D], context lengths L_b ~ U{ctx_lo..ctx_hi}.
    Derived (no draws): q_pos = L_b-1 (the new token's position),
    n_entries = floor(L_b/m), raw_pos0 = L_b-W, raw_len = W (SWA slot j holds
    position L_b-W+j)."""
    B = w.B if B is None else B
    N_cap = w.N_cap if N_cap is None else N_cap
    lo = w.ctx_lo if ctx_lo is None else ctx_lo
    hi = w.ctx_hi if ctx_hi is None else ctx_hi
    g = torch.Generator().manual_seed(seed)
    H, D, H_I, d_I, W = w.H, w.D, w.H_I, w.d_I, w.window
    q = _randn(g, (B, 1, H, D))
    kv_c = _randn(g, (B, N_cap, D))
    qI = _randn(g, (B, 1, H_I, d_I))
    kI_rows = _randn(g, (B, N_cap, d_I))
    swa = _randn(g, (B, W, D))
    L = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64)
    kI_codes, kI_scale = _encode_rows_e4m3(kI_rows)
    dt = torch_dtype(w.dtype)
    L32 = L.to(torch.int32)
    return dict(q=q.to(dt), kv_c=kv_c.to(dt), qI=qI.to(torch.bfloat16), kI_c=kI_codes,
                kI_scale=kI_scale, swa=swa.to(dt), ctx_len=L32,
                q_pos=(L32 - 1).reshape(B, 1).contiguous(),
                n_entries=torch.clamp(L32 // w.m, max=N_cap).to(torch.int32),
                raw_pos0=(L32 - W).to(torch.int32), raw_len=torch.full((B,), W, dtype=torch.int32))


def hca_decode_inputs(w: Workload, seed: int = 0, B: int | None = None, N_cap: int | None = None,
                      ctx: int | None = None):
    """Inputs of one HCA decode step.  Draw order: q [B,1,H,D],
    kv_c cache [B,N_cap,D], SWA cache [B,W,D].  Every element has context
    ``ctx`` (2^20 by default): q_pos = ctx-1, n_entries = floor(ctx/m),
    raw_pos0 = ctx-W, raw_len = W."""
    B = w.B if B is None else B
    N_cap = w.N_cap if N_cap is None else N_cap
    ctx = w.ctx_lo if ctx is None else ctx
    g = torch.Generator().manual_seed(seed)
    H, D, W = w.H, w.D, w.window
    q = _randn(g, (B, 1, H, D))
    kv_c = _randn(g, (B, N_cap, D))
    swa = _randn(g, (B, W, D))
    dt = torch_dtype(w.dtype)
    return dict(q=q.to(dt), kv_c=kv_c.to(dt), swa=swa.to(dt),
                q_pos=torch.full((B, 1), ctx - 1, dtype=torch.int32),
                n_entries=torch.full((B,), min(ctx // w.m, N_cap), dtype=torch.int32),
                raw_pos0=torch.full((B,), ctx - W, dtype=torch.int32),
                raw_len=torch.full((B,), W, dtype=torch.int32))


def hca_prefill_inputs(w: Workload, seed: int = 0, n: int | None = None, B: int | None = None):
    """Inputs of an HCA prefill.  Draw order: q [B,n,H,D], kv [B,n,D],
    W_c ~ N(0, 1/D) [D,D]."""
    n = w.n if n is None else n
    B = w.B if B is None else B
    g = torch.Generator().manual_seed(seed)
    q = _randn(g, (B, n, w.H, w.D))
    kv = _randn(g, (B, n, w.D))
    W_c = _randn(g, (w.D, w.D), 1.0 / math.sqrt(w.D))
    dt = torch_dtype(w.dtype)
    return dict(q=q.to(dt), kv=kv.to(dt), W_c=W_c.to(dt))


def varlen_lengths(total: int, S: int, multiple: int = 4, seed: int = 0) -> list[int]:
    """A length mix for packed prefill: S weights ~ U(0.25, 1.75) scaled to
    total tokens, rounded down to a multiple, the remainder given to the last
    sequence."""
    g = torch.Generator().manual_seed(seed)
    w = 0.25 + 1.5 * torch.rand(S, generator=g, dtype=torch.float64)
    lens = [int(x) // multiple * multiple for x in (w / w.sum() * total).tolist()]
    lens[-1] += total - sum(lens)
    return lens


def indexer_variant_inputs(B: int, n: int, H_I: int, seed: int = 0):
    """Gate weights for the gated indexer: w [B, n, H_I] ~ N(0, 1) (any sign;
    the pages give no distribution)."""
    g = torch.Generator().manual_seed(seed)
    return dict(qI_weight=_randn(g, (B, n, H_I)))


def gated_compressor_weights(d_in: int, d_out: int, m: int, overlap: bool, dtype="bf16",
                             seed: int = 0):
    """Weights of the gated-softmax compressor.  Draw order: W_kv, W_gate
    [d_in, c*d_out] ~ N(0, 1/d_in), ape [m, c*d_out] ~ N(0, 1) (fp32);
    c = 2 if overlap else 1."""
    c = 2 if overlap else 1
    g = torch.Generator().manual_seed(seed)
    W_kv = _randn(g, (d_in, c * d_out), 1.0 / math.sqrt(d_in))
    W_gate = _randn(g, (d_in, c * d_out), 1.0 / math.sqrt(d_in))
    ape = _randn(g, (m, c * d_out))
    dt = torch_dtype(dtype)
    return dict(W_kv=W_kv.to(dt), W_gate=W_gate.to(dt), ape=ape)


def query_sample(n: int, m: int, window: int, count: int, seed: int = 1) -> torch.Tensor:
    """A fixed, seeded subset of query positions for sampled checks at full
    size: positions 0..m, the block boundaries around the first few entries,
    window-1/window/window+1, the last 64 positions, then uniform draws."""
    must = set(range(min(n, m + 1)))
    for i in range(1, 9):
        for d in (-1, 0, 1):
            p = m * i + d
            if 0 <= p < n:
                must.add(p)
    for p in (window - 1, window, window + 1):
        if 0 <= p < n:
            must.add(p)
    must.update(range(max(0, n - 64), n))
    g = torch.Generator().manual_seed(seed)
    rest = torch.randperm(n, generator=g).tolist()
    out = set(must)
    for p in rest:
        if len(out) >= count:
            break
        out.add(p)
    return torch.tensor(sorted(out), dtype=torch.int64)
