"""Bounded device waits: a wait on a barrier that nothing completes ends after its
limit with BCA_ERR_DEVICE_TIMEOUT in the status word, and the context stays usable."""
import os

import pytest
import torch

import block_causal_attention_dit_b200 as bca

pytestmark = pytest.mark.gpu


def test_wait_expires_with_status(cuda_device):
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bca.selftest_wait_timeout(status, 5_000_000)
    torch.cuda.synchronize()
    got = int(status.item())
    # The self-checking build (BCA_DEVICE_CHECKS) records 1000 + the wait's site.
    checked = "checked" in os.path.basename(bca.LIB_PATH)
    assert got == 6 or (checked and 1000 <= got < 2000), got
    # the context is still usable
    x = torch.ones(4, device=cuda_device)
    assert float((x * 2).sum().item()) == 8.0
