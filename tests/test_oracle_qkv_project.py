"""Pins of the oracle's Q/K/V projection with the Q/K norm and rotary embedding
("SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll", "Siffrorna, och vad de inte
säger": the Q/K-norm change between the projection of the target rows and the
attention; reading: y = x w^T with w in the torch Linear layout [Q heads | K heads |
V heads], then rope(rms_norm(.)) of every Q and K head vector, V as projected).

Each pin checks the function against something other than itself:
  * the V part against numpy's fp64 matmul (a library routine the oracle does not
    call);
  * identity weight blocks reduce Q and K to the already pinned rms_norm + rope of
    the input rows, bit for bit, and V to the input itself -- this fixes which
    output features feed Q, K and V and which weight vector each uses;
  * a permutation and a head rotation in the weights fix the orientation of w
    (row n of w is output feature n) and the head order;
  * a selection of rows equals those rows of the full result."""
import numpy as np
import pytest
import torch

import oracle

d = 128


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _tables(T, seed):
    rng = np.random.default_rng(seed)
    ang = rng.uniform(-np.pi, np.pi, (T, d // 2))
    gq = rng.uniform(0.5, 1.5, d).astype(np.float32)
    gk = rng.uniform(0.5, 1.5, d).astype(np.float32)
    return gq, gk, np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def _x(T, D, seed):
    return _bf16(np.random.default_rng(seed).standard_normal((T, D)))


def test_v_part_is_the_matrix_product():
    T, D, H = 9, 96, 2
    x = _x(T, D, 1)
    w = _bf16(np.random.default_rng(2).standard_normal((3 * H * d, D)) * 0.1)
    gq, gk, c, s = _tables(T, 3)
    q, k, v = oracle.qkv_project(x, w, gq, gk, c, s, 1e-6, H)
    y = x.double().numpy() @ w.double().numpy().T
    np.testing.assert_allclose(v.reshape(T, H * d), y[:, 2 * H * d:], rtol=1e-12, atol=1e-12)
    # Q and K are the norm + rotary of their blocks of the same product
    yq = y[:, :H * d].reshape(T, H, d)
    inv = 1.0 / np.sqrt((yq ** 2).mean(-1, keepdims=True) + 1e-6)
    n = yq * inv * gq.astype(np.float64)
    cc, ss = c.astype(np.float64)[:, None, :], s.astype(np.float64)[:, None, :]
    want = np.empty_like(n)
    want[..., 0::2] = n[..., 0::2] * cc - n[..., 1::2] * ss
    want[..., 1::2] = n[..., 0::2] * ss + n[..., 1::2] * cc
    np.testing.assert_allclose(q, want, rtol=1e-10, atol=1e-12)


def _identity_blocks(H, scales=(1.0, 1.0, 1.0)):
    D = H * d
    eye = np.eye(D, dtype=np.float32)
    return _bf16(np.concatenate([scales[0] * eye, scales[1] * eye, scales[2] * eye]))


def test_identity_weights_reduce_to_the_pinned_norm_and_rope():
    T, H = 7, 3
    x = _x(T, H * d, 4)
    gq, gk, c, s = _tables(T, 5)
    q, k, v = oracle.qkv_project(x, _identity_blocks(H), gq, gk, c, s, 1e-6, H)
    xh = x.view(T, H, d)
    assert np.array_equal(q, oracle.qk_norm_rope(xh, gq, c, s, 1e-6))
    assert np.array_equal(k, oracle.qk_norm_rope(xh, gk, c, s, 1e-6))
    assert np.array_equal(v, xh.double().numpy())
    assert not np.array_equal(q, k)  # the two weight vectors differ


def test_v_block_scaled_and_norm_scale_invariant():
    """W_v = 2I doubles V exactly; W_q = 4I leaves Q unchanged at eps = 0 (the RMS
    norm removes the scale: 4 is a power of two, so the fp64 values are equal)."""
    T, H = 5, 2
    x = _x(T, H * d, 6)
    gq, gk, c, s = _tables(T, 7)
    q1, _, v1 = oracle.qkv_project(x, _identity_blocks(H), gq, gk, c, s, 0.0, H)
    q4, _, v2 = oracle.qkv_project(x, _identity_blocks(H, (4.0, 1.0, 2.0)), gq, gk, c, s, 0.0, H)
    assert np.array_equal(v2, 2.0 * v1)
    assert np.array_equal(q4, q1)


def test_weight_orientation_and_head_order():
    """Q block = a permutation P (row n of w picks input channel perm[n]): Q equals
    the norm + rotary of x[:, perm], which differs from x[:, argsort(perm)] (the
    transposed reading).  Rotating the Q block by one head moves the heads."""
    T, H = 4, 2
    D = H * d
    x = _x(T, D, 8)
    gq, gk, c, s = _tables(T, 9)
    perm = np.random.default_rng(10).permutation(D)
    P = np.zeros((D, D), dtype=np.float32)
    P[np.arange(D), perm] = 1.0
    eye = np.eye(D, dtype=np.float32)
    w = _bf16(np.concatenate([P, eye, eye]))
    q, _, _ = oracle.qkv_project(x, w, gq, gk, c, s, 1e-6, H)
    xp = x[:, torch.from_numpy(perm)].contiguous().view(T, H, d)
    assert np.array_equal(q, oracle.qk_norm_rope(xp, gq, c, s, 1e-6))
    xt = x[:, torch.from_numpy(np.argsort(perm))].contiguous().view(T, H, d)
    assert not np.allclose(q, oracle.qk_norm_rope(xt, gq, c, s, 1e-6))
    rot = np.roll(eye, d, axis=0)  # output head h reads input head h - 1
    q2, _, _ = oracle.qkv_project(x, _bf16(np.concatenate([rot, eye, eye])), gq, gk, c, s, 1e-6, H)
    want = oracle.qk_norm_rope(x.view(T, H, d)[:, [H - 1] + list(range(H - 1))].contiguous(),
                               gq, c, s, 1e-6)
    assert np.array_equal(q2, want)


def test_selected_rows_equal_full_rows():
    T, D, H = 11, 64, 1
    x = _x(T, D, 11)
    w = _bf16(np.random.default_rng(12).standard_normal((3 * H * d, D)) * 0.2)
    gq, gk, c, s = _tables(T, 13)
    full = oracle.qkv_project(x, w, gq, gk, c, s, 1e-6, H)
    rows = [10, 0, 3]
    part = oracle.qkv_project(x, w, gq, gk, c, s, 1e-6, H, rows=rows)
    for a, b in zip(full, part):
        assert np.array_equal(a[rows], b)
    with pytest.raises(ValueError):
        oracle.qkv_project(x, w, gq, gk, c, s, 1e-6, H, rows=[T])
