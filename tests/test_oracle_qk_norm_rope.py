"""Pins for the oracle's Q/K RMS norm and rotary embedding (the steps next to the
attention; "SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll", "Siffrorna, och
vad de inte säger", names the Q/K norm; the formula is the plain reading: RMS
norm over the head dimension with a weight vector, then consecutive channel pairs
turned by per-row angles).

Checked against: PyTorch's rms_norm (a library routine sharing nothing with this
repo), complex multiplication by e^{i theta} in numpy (the rotation's definition),
a closed form for constant vectors, scale invariance, the direction of a quarter
turn, norm preservation and undoing a turn."""
import math

import numpy as np
import torch

import oracle

D = 128


def _x(rows, H, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, H, D, generator=g) * scale).to(torch.bfloat16)


def _tables(rows, seed):
    rng = np.random.default_rng(seed)
    ang = rng.uniform(-math.pi, math.pi, (rows, D // 2))
    return ang, np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def test_norm_matches_torch_rms_norm():
    x = _x(37, 3, 1, scale=2.5)
    gamma = np.random.default_rng(2).uniform(0.5, 1.5, D).astype(np.float32)
    for eps in (1e-6, 1e-2):
        got = oracle.rms_norm(x, gamma, eps)
        want = torch.nn.functional.rms_norm(x.double(), (D,), torch.from_numpy(gamma).double(),
                                            eps).numpy()
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)


def test_norm_closed_form_and_scale_invariance():
    gamma = np.random.default_rng(3).uniform(0.5, 1.5, D).astype(np.float32)
    for c in (0.75, -3.0, 1e-3):
        x = torch.full((1, 1, D), c, dtype=torch.bfloat16)
        cb = float(x[0, 0, 0])
        got = oracle.rms_norm(x, gamma, 1e-6)[0, 0]
        want = gamma.astype(np.float64) * cb / math.sqrt(cb * cb + 1e-6)
        np.testing.assert_allclose(got, want, rtol=1e-14)
    x = _x(5, 2, 4)
    np.testing.assert_array_equal(oracle.rms_norm(x * 2, gamma, 0.0), oracle.rms_norm(x, gamma, 0.0))


def test_rope_is_complex_multiplication():
    rows, H = 9, 2
    ang, c, s = _tables(rows, 5)
    y = np.random.default_rng(6).normal(size=(rows, H, D))
    got = oracle.rope(y, c, s)
    z = y[..., 0::2] + 1j * y[..., 1::2]
    w = z * (c.astype(np.float64) + 1j * s.astype(np.float64))[:, None, :]
    want = np.empty_like(y)
    want[..., 0::2], want[..., 1::2] = w.real, w.imag
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-14)


def test_rope_quarter_turn_direction():
    y = np.zeros((1, 1, D))
    y[0, 0, 0::2] = 1.0  # every pair is (1, 0)
    c = np.zeros((1, D // 2), np.float32)
    s = np.ones((1, D // 2), np.float32)
    out = oracle.rope(y, c, s)
    assert np.all(out[0, 0, 0::2] == 0.0) and np.all(out[0, 0, 1::2] == 1.0)  # (1,0) -> (0,1)


def test_rope_preserves_pair_norms_and_undoes():
    rows, H = 11, 3
    _, c, s = _tables(rows, 7)
    y = np.random.default_rng(8).normal(size=(rows, H, D))
    out = oracle.rope(y, c, s)
    k = (c.astype(np.float64) ** 2 + s.astype(np.float64) ** 2)[:, None, :]
    n_in = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    n_out = out[..., 0::2] ** 2 + out[..., 1::2] ** 2
    np.testing.assert_allclose(n_out, n_in * k, rtol=1e-12)
    back = oracle.rope(out, c, -s)
    np.testing.assert_allclose(back, y * k.repeat(2, axis=-1), rtol=1e-12, atol=1e-12)


def test_identity_angles_reduce_to_the_norm():
    x = _x(6, 4, 9)
    gamma = np.random.default_rng(10).uniform(0.5, 1.5, D).astype(np.float32)
    c = np.ones((6, D // 2), np.float32)
    s = np.zeros((6, D // 2), np.float32)
    np.testing.assert_array_equal(oracle.qk_norm_rope(x, gamma, c, s, 1e-6),
                                  oracle.rms_norm(x, gamma, 1e-6))
