"""Failure detection on the GPU without a fault: the bounded-wait path.

A barrier that nothing completes makes one warp's wait give up after a short
limit; the library records it and csa_check reports CSA_ERR_TIMEOUT once, the
record is cleared, and the context stays usable for the layer's kernels."""
import pytest
import torch

import compressed_sparse_attention_11_b200 as csa

pytestmark = pytest.mark.gpu


def test_completed_barrier_is_not_a_timeout():
    assert csa.selftest_wait(20000, arrive=True) == csa.CSA_OK


def test_expired_wait_is_reported_once_and_context_survives():
    assert csa.selftest_wait(20000, arrive=False) == csa.CSA_ERR_TIMEOUT
    csa.csa_check()  # the record was cleared by the first check
    x = torch.randn(1, 64, 16, device="cuda")
    b = torch.zeros(4, 16, device="cuda")
    out = csa.csa_compress(x, x, x, x, b, b, 4)
    torch.cuda.synchronize()
    csa.csa_check()
    assert torch.isfinite(out).all()
