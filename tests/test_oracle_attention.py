"""Pins for the oracle's attention: each test checks it against something other
than itself -- a direct numpy evaluation with an explicit mask matrix, PyTorch's
scaled_dot_product_attention in fp64 for the special cases that reduce to plain
full or plain causal attention, closed forms, and the invariants the pages fix
("Serving architecture: the cross-step prefix KV cache": prefix K/V computed in
step 1 is exact for later steps, because prefix blocks never see the target)."""
import math

import numpy as np
import pytest
import torch

import oracle


def rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def f64(x):
    return x.to(torch.float64).numpy()


def offsets_of(blocks):
    return np.concatenate([[0], np.cumsum(blocks)]).astype(np.int32)


def brute_force(q, k, v, blocks, scale):
    """Explicit S x S mask matrix and a direct softmax, per head, in numpy fp64."""
    Q, K, V = f64(q), f64(k), f64(v)
    S, H, d = Q.shape
    blk = np.repeat(np.arange(len(blocks)), blocks)
    allowed = blk[None, :] <= blk[:, None]  # block of key <= block of query
    out = np.zeros_like(Q)
    for h in range(H):
        s = (Q[:, h, :] @ K[:, h, :].T) * scale
        s = np.where(allowed, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ V[:, h, :]
    return out


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    S = int(rng.integers(1, 17))
    H = int(rng.integers(1, 3))
    d = int(rng.integers(4, 9))
    # random split of S into 1..S ordered blocks
    n_blocks = int(rng.integers(1, S + 1))
    cuts = np.sort(rng.choice(np.arange(1, S), size=n_blocks - 1, replace=False)) if n_blocks > 1 else []
    blocks = np.diff(np.concatenate([[0], cuts, [S]])).astype(int)
    q, k, v = (rand_bf16((S, H, d), seed * 10 + t, 1.5) for t in range(3))
    scale = 1.0 / math.sqrt(d)
    got = oracle.prefill(q, k, v, offsets_of(blocks), scale)
    want = brute_force(q, k, v, blocks, scale)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def test_single_block_is_full_attention_sdpa():
    S, H, d = 48, 3, 16
    q, k, v = (rand_bf16((S, H, d), 100 + t) for t in range(3))
    scale = 0.37
    got = oracle.prefill(q, k, v, [0, S], scale)
    tq, tk, tv = (x.to(torch.float64).permute(1, 0, 2) for x in (q, k, v))
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    np.testing.assert_allclose(got, want.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_unit_blocks_are_causal_attention_sdpa():
    S, H, d = 40, 2, 8
    q, k, v = (rand_bf16((S, H, d), 200 + t) for t in range(3))
    scale = 1.0 / math.sqrt(d)
    got = oracle.prefill(q, k, v, np.arange(S + 1), scale)
    tq, tk, tv = (x.to(torch.float64).permute(1, 0, 2) for x in (q, k, v))
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                            scale=scale)
    np.testing.assert_allclose(got, want.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_zero_query_gives_mean_of_allowed_values():
    """q = 0 makes every allowed score equal, so row i's output is the plain mean
    of V over keys [0, end of its block): pins every block boundary."""
    blocks = [5, 3, 7, 1, 4]
    S, H, d = sum(blocks), 2, 6
    q = torch.zeros((S, H, d), dtype=torch.bfloat16)
    k, v = rand_bf16((S, H, d), 1), rand_bf16((S, H, d), 2)
    got = oracle.prefill(q, k, v, offsets_of(blocks), 0.5)
    ends = np.repeat(offsets_of(blocks)[1:], blocks)
    V = f64(v)
    for i in range(S):
        np.testing.assert_allclose(got[i], V[: ends[i]].mean(axis=0), rtol=1e-13, atol=1e-15)


def test_constant_values_give_constant_output():
    blocks = [4, 9, 3]
    S, H, d = sum(blocks), 2, 5
    q, k = rand_bf16((S, H, d), 3), rand_bf16((S, H, d), 4)
    v = torch.full((S, H, d), -2.75, dtype=torch.bfloat16)
    got = oracle.prefill(q, k, v, offsets_of(blocks), 0.8)
    np.testing.assert_allclose(got, -2.75, rtol=1e-14)


def test_identical_keys_give_uniform_average():
    blocks = [6, 2, 5]
    S, H, d = sum(blocks), 1, 4
    q, v = rand_bf16((S, H, d), 5), rand_bf16((S, H, d), 6)
    k = rand_bf16((1, H, d), 7).expand(S, H, d).contiguous()
    got = oracle.prefill(q, k, v, offsets_of(blocks), 1.0)
    ends = np.repeat(offsets_of(blocks)[1:], blocks)
    V = f64(v)
    for i in range(S):
        np.testing.assert_allclose(got[i], V[: ends[i]].mean(axis=0), rtol=1e-13, atol=1e-15)


def test_rows_are_probability_vectors():
    """With V[j] = e_j (one-hot, d = S) the output row is the softmax row itself:
    entries are >= 0, masked keys are exactly 0, and each row sums to 1."""
    blocks = [3, 5, 4]
    S = sum(blocks)
    H, d = 2, S
    q, k = rand_bf16((S, H, d), 8, 2.0), rand_bf16((S, H, d), 9, 2.0)
    v = torch.zeros((S, H, d), dtype=torch.bfloat16)
    for j in range(S):
        v[j, :, j] = 1.0
    P = oracle.prefill(q, k, v, offsets_of(blocks), 0.3)
    ends = np.repeat(offsets_of(blocks)[1:], blocks)
    assert (P >= 0).all()
    for i in range(S):
        assert np.all(P[i, :, ends[i]:] == 0.0)
        assert np.all(P[i, :, : ends[i]] > 0.0)
    np.testing.assert_allclose(P.sum(axis=2), 1.0, rtol=0, atol=1e-12)


def _split(x, P):
    return x[:P], x[P:]


def test_cached_step_equals_full_recompute_bitwise():
    """The target rows of a block-causal pass over [prefix ; target] equal a cached
    step that reads the prefix K/V from a [H, cap, d] cache: same keys, same order."""
    blocks = [7, 12, 5, 9]
    S, H, d = sum(blocks), 3, 8
    q, k, v = (rand_bf16((S, H, d), 20 + t) for t in range(3))
    P = S - blocks[-1]
    full = oracle.prefill(q, k, v, offsets_of(blocks), 0.4)
    cap = P + 3  # a slot larger than the prefix: stale rows must not be read
    kc = torch.full((H, cap, d), float("nan"), dtype=torch.bfloat16)
    vc = torch.full((H, cap, d), float("nan"), dtype=torch.bfloat16)
    kc[:, :P] = k[:P].permute(1, 0, 2)
    vc[:, :P] = v[:P].permute(1, 0, 2)
    step = oracle.cached_step(q[P:], k[P:], v[P:], kc, vc, P, 0.4)
    assert np.array_equal(step, full[P:])


def test_prefix_rows_do_not_see_the_target():
    blocks = [6, 10, 8]
    S, H, d = sum(blocks), 2, 8
    q, k, v = (rand_bf16((S, H, d), 30 + t) for t in range(3))
    P = S - blocks[-1]
    a = oracle.prefill(q, k, v, offsets_of(blocks), 0.5)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    for x, s in ((q2, 40), (k2, 41), (v2, 42)):
        x[P:] = rand_bf16((S - P, H, d), s, 3.0)
    b = oracle.prefill(q2, k2, v2, offsets_of(blocks), 0.5)
    assert np.array_equal(a[:P], b[:P])
    assert not np.allclose(a[P:], b[P:])


def test_selected_rows_match_all_rows():
    blocks = [9, 4, 11]
    S, H, d = sum(blocks), 2, 8
    q, k, v = (rand_bf16((S, H, d), 50 + t) for t in range(3))
    full = oracle.prefill(q, k, v, offsets_of(blocks), 0.5)
    rows = [23, 0, 8, 9, 12, 13]
    part = oracle.prefill(q, k, v, offsets_of(blocks), 0.5, rows=rows)
    assert np.array_equal(part, full[rows])
    P = S - blocks[-1]
    kc = k[:P].permute(1, 0, 2).contiguous()
    vc = v[:P].permute(1, 0, 2).contiguous()
    st = oracle.cached_step(q[P:], k[P:], v[P:], kc, vc, P, 0.5)
    st_rows = oracle.cached_step(q[P:], k[P:], v[P:], kc, vc, P, 0.5, rows=[10, 0, 3])
    assert np.array_equal(st_rows, st[[10, 0, 3]])


def test_no_prefix_is_plain_attention():
    """P = 0: the cached step reduces to full attention over the target alone."""
    T, H, d = 21, 2, 8
    q, k, v = (rand_bf16((T, H, d), 60 + t) for t in range(3))
    empty = torch.zeros((H, 0, d), dtype=torch.bfloat16)
    got = oracle.cached_step(q, k, v, empty, empty, 0, 0.6)
    tq, tk, tv = (x.to(torch.float64).permute(1, 0, 2) for x in (q, k, v))
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.6)
    np.testing.assert_allclose(got, want.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_cached_step_against_brute_force_with_e4m3_cache():
    """e4m3 cache entries are read as fp32(decode(code) * scale): compare with a
    direct numpy evaluation over explicitly dequantised keys/values."""
    T, P, H, d = 9, 13, 2, 8
    q, k, v = (rand_bf16((T, H, d), 70 + t) for t in range(3))
    rng = np.random.default_rng(7)
    codes_k = rng.integers(0, 256, size=(H, P, d), dtype=np.uint8)
    codes_v = rng.integers(0, 256, size=(H, P, d), dtype=np.uint8)
    for c in (codes_k, codes_v):  # no NaN codes
        c[(c & 0x7F) == 0x7F] = 0x3A
    ks = np.array([0.013, 0.5], dtype=np.float32)
    vs = np.array([0.02, 1.75], dtype=np.float32)
    got = oracle.cached_step(q, k, v, codes_k, codes_v, P, 0.35, k_kind=oracle.KIND_E4M3,
                             v_kind=oracle.KIND_E4M3, k_scale=ks, v_scale=vs)
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    Kc = (table[codes_k] * ks[:, None, None]).astype(np.float32).astype(np.float64)
    Vc = (table[codes_v] * vs[:, None, None]).astype(np.float32).astype(np.float64)
    Q, K, V = f64(q), f64(k), f64(v)
    for h in range(H):
        keys = np.concatenate([Kc[h], K[:, h]], axis=0)
        vals = np.concatenate([Vc[h], V[:, h]], axis=0)
        s = Q[:, h] @ keys.T * 0.35
        p = np.exp(s - s.max(axis=1, keepdims=True))
        want = (p / p.sum(axis=1, keepdims=True)) @ vals
        np.testing.assert_allclose(got[:, h], want, rtol=1e-12, atol=1e-13)


def test_power_of_two_scaled_e4m3_cache_equals_bf16_cache():
    """Every e4m3 value times a power of two is exactly a bf16 value, so an e4m3
    cache with scale 2^k must give bit-identical results to the same values held
    as a bf16 cache (pins indexing and dequantisation of 1-byte rows)."""
    T, P, H, d = 7, 11, 2, 8
    q, k, v = (rand_bf16((T, H, d), 80 + t) for t in range(3))
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 256, size=(2, H, P, d), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x41
    scales = np.array([0.25, 8.0], dtype=np.float32)
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32)
    bf = [(table[torch.from_numpy(codes[i].astype(np.int64))] * torch.from_numpy(scales)[:, None, None]
           ).to(torch.bfloat16) for i in range(2)]
    a = oracle.cached_step(q, k, v, codes[0], codes[1], P, 0.5, k_kind=oracle.KIND_E4M3,
                           v_kind=oracle.KIND_E4M3, k_scale=scales, v_scale=scales)
    b = oracle.cached_step(q, k, v, bf[0], bf[1], P, 0.5)
    assert np.array_equal(a, b)


def test_bad_arguments_are_rejected():
    q = rand_bf16((8, 1, 4), 1)
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, [0, 3, 3, 8], 1.0)  # empty block
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, [0, 9], 1.0)  # does not end at S
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, [0, 8], 1.0, rows=[8])
