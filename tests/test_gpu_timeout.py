"""Bounded device waits: a wait on a barrier that nothing completes ends after its
limit with BCA_ERR_DEVICE_TIMEOUT in the status word, and the context stays usable."""
import pytest
import torch

import block_causal_attention_dit_b200 as bca

pytestmark = pytest.mark.gpu


def test_wait_expires_with_status(cuda_device):
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bca.selftest_wait_timeout(status, 5_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == 6
    # the context is still usable
    x = torch.ones(4, device=cuda_device)
    assert float((x * 2).sum().item()) == 8.0


def test_software_exp2_error_bound(cuda_device):
    """The FMA-pipe 2^x used for part of every softmax row: relative error within
    the fitted polynomial's bound (7.5e-5, checked at 1e-4) against exact 2^x for
    normal results, and exactly 0 for x <= -127 (masked keys must contribute 0)."""
    import numpy as np
    xs = np.concatenate([np.linspace(-126.0, 8.0, 200001), [-0.5, 0.5, 0.0, 7.999, -1e-7],
                         np.random.default_rng(0).uniform(-30, 8, 100000)]).astype(np.float32)
    x = torch.from_numpy(xs).to(cuda_device)
    yp, ym = bca.selftest_exp2(x)
    torch.cuda.synchronize()
    want = np.exp2(xs.astype(np.float64))
    got = yp.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - want) <= 1e-4 * want)
    # the hardware ex2 it stands in for is within the same bound
    assert np.all(np.abs(ym.cpu().numpy() - want) <= 1e-4 * want)
    zero_in = torch.tensor([-127.0, -127.4, -200.0, -1e30, float("-inf")], device=cuda_device)
    z, _ = bca.selftest_exp2(zero_in)
    assert torch.all(z == 0)
