"""Failure paths on the GPU without a fault, trap or hang: a launch failure
injected after validation is reported as CSA_ERR_CUDA, once."""
import pytest
import torch

from long_context_compressed_03_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_injected_launch_failure_is_reported_and_one_shot():
    x = torch.randn(1, 64, 32, device=DEV)
    W = torch.randn(32, 32, device=DEV)
    lib = api.load()
    assert lib.csa_debug_inject_launch_error(719) == api.CSA_OK
    with pytest.raises(api.CsaError) as ei:
        api.compress(x, W, 4, True)
    assert ei.value.status == api.CSA_ERR_CUDA
    out = api.compress(x, W, 4, True)                # the next call launches
    torch.cuda.synchronize()
    assert out.shape == (1, 16, 32) and torch.isfinite(out).all()


# The timeout path: a short wait limit and a stalled launch (one thread of
# every CTA waits on a barrier nothing completes) make a bounded wait run out.
# The kernel records CSA_ERR_TIMEOUT and its CTAs drain what they issued and
# exit; the check reports the timeout once, and the next call runs clean.
def _attn_case():
    g = torch.Generator().manual_seed(11)
    n, N_c, k = 512, 128, 64
    q = torch.randn(1, n, 64, 128, generator=g).to(torch.bfloat16).to(DEV)
    kv = torch.randn(1, n, 128, generator=g).to(torch.bfloat16).to(DEV)
    kv_c = torch.randn(1, N_c, 128, generator=g).to(torch.bfloat16).to(DEV)
    idx = torch.randint(0, N_c, (1, n, k), generator=g, dtype=torch.int32).to(DEV)
    return q, kv, kv_c, idx


def _expect_timeout_then_clean(run):
    lib = api.load()
    api.csa_check_device_error()                     # nothing pending
    ref = run()
    torch.cuda.synchronize()
    assert lib.csa_debug_set_wait_limit(2_000_000, 1) == api.CSA_OK      # 2 ms, stall next
    try:
        run()
        with pytest.raises(api.CsaError) as ei:
            api.csa_check_device_error(clear=True)
        assert ei.value.status == api.CSA_ERR_TIMEOUT
    finally:
        assert lib.csa_debug_set_wait_limit(0, 0) == api.CSA_OK
    api.csa_check_device_error()                     # cleared
    again = run()
    torch.cuda.synchronize()
    api.csa_check_device_error()
    assert torch.equal(again, ref)


def test_attention_wait_timeout_is_reported_and_the_next_call_runs_clean():
    q, kv, kv_c, idx = _attn_case()
    _expect_timeout_then_clean(lambda: api.sparse_attn(q, kv_c, idx, kv, 128))


def test_indexer_wait_timeout_is_reported_and_the_next_call_runs_clean():
    g = torch.Generator().manual_seed(12)
    n = 4096
    qI = torch.randn(1, n, 4, 64, generator=g).to(torch.bfloat16).to(DEV)
    kI = torch.randn(1, n // 4, 64, generator=g).to(torch.bfloat16).to(DEV)
    _expect_timeout_then_clean(lambda: api.indexer_topk(qI, kI, 4, 64))


def test_decode_attention_wait_timeout_is_reported_and_the_next_call_runs_clean():
    # decode rows (positions given): the tcgen05 decode kernel with its TMA
    # window tiles and gathered entry tiles in flight when the wait runs out
    g = torch.Generator().manual_seed(13)
    B, N_cap, k, W = 4, 4000, 512, 256
    q = torch.randn(B, 1, 64, 128, generator=g).to(torch.bfloat16).to(DEV)
    kv_c = torch.randn(B, N_cap, 128, generator=g).to(torch.bfloat16).to(DEV)
    swa = torch.randn(B, W, 128, generator=g).to(torch.bfloat16).to(DEV)
    ctx = torch.tensor([16000, 9000, 12345, 700], dtype=torch.int32)
    idx = torch.full((B, k), -1, dtype=torch.int32)
    for b in range(B):
        sel = torch.randperm(min(int(ctx[b]) // 4, N_cap), generator=g)[:k]
        idx[b, :sel.numel()] = sel.to(torch.int32)
    kw = dict(raw_pos0=(ctx - W).to(DEV), raw_len=torch.full((B,), W, dtype=torch.int32).to(DEV),
              q_pos=(ctx - 1).reshape(B, 1).to(DEV))
    idx = idx.reshape(B, 1, k).to(DEV)
    _expect_timeout_then_clean(lambda: api.sparse_attn(q, kv_c, idx, swa, W, **kw))

