"""Bounded-wait give-up path on the GPU: a barrier nothing completes makes the
wait run out, the kernel records the timeout and returns, and the context
stays usable. No fault, trap or hang is involved."""
import pytest
import torch

import global_soft_capped_b200 as g2

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert g2.g2attn_selftest_wait_timeout(10000) == g2.G2ATTN_ERR_DEVICE_TIMEOUT
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK     # read-and-clear
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0                           # context still usable
