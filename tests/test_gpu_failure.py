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
