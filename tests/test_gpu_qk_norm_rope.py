"""bca_qk_norm_rope against the oracle: every output element is within one bf16
ulp of the exact (fp64) value, plus the fp32 rounding of the rotation (1e-6 of the
pair's magnitude); nearly all are the round-to-nearest-even of it.  The kernel
works in fp32 and rounds once to bf16, so its error is at most half an ulp plus a
few fp32 roundings (~1e-7 relative) -- one ulp bounds it with room, and a wrong
sign, pair, weight or normaliser breaks the bound by orders of magnitude."""
import math

import numpy as np
import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200.workloads import randn_bf16

pytestmark = pytest.mark.gpu
D = 128


def _inputs(rows, H, device, seed, scale=1.0):
    q = (randn_bf16((rows, H, D), seed, device).float() * scale).to(torch.bfloat16)
    k = (randn_bf16((rows, H, D), seed + 1, device).float() * scale + 0.5).to(torch.bfloat16)
    rng = np.random.default_rng(seed)
    gq = rng.uniform(0.5, 1.5, D).astype(np.float32)
    gk = rng.uniform(0.5, 1.5, D).astype(np.float32)
    pos = np.arange(rows, dtype=np.float64)[:, None]
    freq = 10000.0 ** (-np.arange(D // 2, dtype=np.float64) / (D // 2))
    ang = pos * freq + rng.uniform(-0.1, 0.1, (rows, D // 2))
    c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).to(device)
    return q, k, gq, gk, c, s, dev


def _ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _check(got, x, gamma, c, s, eps, rows=None, what=""):
    xb = x.cpu() if rows is None else x.cpu()[rows]
    cc, ss = (c, s) if rows is None else (c[rows], s[rows])
    y = oracle.rms_norm(xb, gamma, eps)
    want = oracle.rope(y, cc, ss)
    g = got.cpu().double().numpy() if rows is None else got.cpu()[rows].double().numpy()
    mag = np.sqrt(y[..., 0::2] ** 2 + y[..., 1::2] ** 2).repeat(2, axis=-1)
    err = np.abs(g - want)
    bound = _ulp_bf16(want) + 1e-6 * mag
    assert np.all(err <= bound), f"{what}: worst excess {np.max(err - bound):.3e}"
    rne = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
    assert np.mean(g == rne) > 0.99, what


@pytest.mark.parametrize("rows,H,scale", [(300, 4, 1.0), (129, 3, 40.0), (64, 2, 1e-2)])
def test_matches_oracle(cuda_device, rows, H, scale):
    q, k, gq, gk, c, s, dev = _inputs(rows, H, cuda_device, 11 + rows, scale)
    q0, k0 = q.clone(), k.clone()
    bca.qk_norm_rope(q, k, dev(gq), dev(gk), dev(c), dev(s), eps=1e-6)
    torch.cuda.synchronize()
    _check(q, q0, gq, c, s, 1e-6, what="q")
    _check(k, k0, gk, c, s, 1e-6, what="k")


def test_one_tensor_only_and_empty(cuda_device):
    q, k, gq, gk, c, s, dev = _inputs(100, 2, cuda_device, 21)
    q0, k0 = q.clone(), k.clone()
    bca.qk_norm_rope(None, k, None, dev(gk), dev(c), dev(s), eps=1e-5)
    torch.cuda.synchronize()
    assert torch.equal(q, q0)
    _check(k, k0, gk, c, s, 1e-5, what="k only")
    e = torch.empty((0, 2, D), dtype=torch.bfloat16, device=cuda_device)
    bca.qk_norm_rope(e, e, dev(gq), dev(gk), dev(c), dev(s))  # rows == 0: nothing to do
    with pytest.raises(bca.BcaError):
        bca.qk_norm_rope(None, None, dev(gq), dev(gk), dev(c), dev(s))


def test_t2i_target_rows_sampled(cuda_device):
    """The T2I cached step's target tensors (4096 rows x 32 heads), sampled rows."""
    rows, H = 4096, 32
    q, k, gq, gk, c, s, dev = _inputs(rows, H, cuda_device, 31)
    q0, k0 = q.clone(), k.clone()
    bca.qk_norm_rope(q, k, dev(gq), dev(gk), dev(c), dev(s), eps=1e-6)
    torch.cuda.synchronize()
    pick = np.unique(np.concatenate([np.random.default_rng(3).integers(0, rows, 200),
                                     [0, 1, rows - 2, rows - 1]]))
    _check(q, q0, gq, c, s, 1e-6, rows=pick, what="t2i q")
    _check(k, k0, gk, c, s, 1e-6, rows=pick, what="t2i k")
