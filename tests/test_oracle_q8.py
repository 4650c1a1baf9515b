"""Pins of the oracle's e4m3-Q reading of the cached step (q8=...): the request's
Q quantised per head with the cache's encoder and scale rule ("Qwen/Qwen-Image-2.1"
vLLM recipe, "Prefix KV cache", applied to Q); the scores against the cached keys
use the dequantised Q, those against the target's own keys the bf16 Q.

Each pin reduces the reading to the plain cached step (itself pinned to SDPA, the
prefill and brute force elsewhere) on inputs where the answer is fixed:
* no cached keys: the quantised Q is never used;
* cached keys all zero: their scores are 0 whatever Q meets them, so only the own
  keys' (bf16) scores matter;
* own keys all zero and every head's absmax 7 (scale 7/448 = 2^-6, so the
  dequantised Q is a bf16 tensor): equal to the plain step run with that tensor as Q.
The last two would fail if the two Q's were swapped between the key sources.
"""
import math

import numpy as np
import torch

import oracle
from block_causal_attention_dit_b200.workloads import randn_bf16

SCALE = 1.0 / math.sqrt(128)


def _inputs(T, P, H, seed):
    q, k, v = (randn_bf16((T, H, 128), seed + i) for i in range(3))
    kc, vc = (randn_bf16((P, H, 128), seed + 3 + i).permute(1, 0, 2).contiguous()
              for i in range(2))
    return q, k, v, kc, vc


def _q8(q):
    return oracle.quantize_prefix(q, q.shape[0])


def test_without_cached_keys_the_plain_step():
    q, k, v, kc, vc = _inputs(37, 1, 2, 10)
    plain = oracle.cached_step(q, k, v, kc, vc, 0, SCALE)
    got = oracle.cached_step(q, k, v, kc, vc, 0, SCALE, q8=_q8(q))
    assert np.array_equal(plain, got)


def test_own_keys_meet_the_bf16_q():
    q, k, v, kc, vc = _inputs(37, 50, 2, 20)
    kc = torch.zeros_like(kc)
    plain = oracle.cached_step(q, k, v, kc, vc, 50, SCALE)
    got = oracle.cached_step(q, k, v, kc, vc, 50, SCALE, q8=_q8(q))
    assert np.array_equal(plain, got)


def test_cached_keys_meet_the_dequantised_q():
    T, P, H = 37, 50, 2
    q, k, v, kc, vc = _inputs(T, P, H, 30)
    q = q.float().clamp(-6.5, 6.5)
    q[3, :, 5] = 7.0  # every head's absmax: scale 7 / 448 = 2^-6 exactly
    q = q.to(torch.bfloat16)
    k = torch.zeros_like(k)
    codes, scales = _q8(q)
    assert np.all(scales == np.float32(2.0 ** -6))
    table = np.array([oracle.e4m3_decode(c) for c in range(256)], dtype=np.float32)
    q_deq = torch.from_numpy(table[codes] * np.float32(2.0 ** -6)).permute(1, 0, 2)
    q_deq_bf16 = q_deq.to(torch.bfloat16)
    assert torch.equal(q_deq_bf16.float(), q_deq)  # e4m3 values x 2^-6 are bf16 values
    got = oracle.cached_step(q, k, v, kc, vc, P, SCALE, q8=(codes, scales))
    want = oracle.cached_step(q_deq_bf16.contiguous(), k, v, kc, vc, P, SCALE)
    assert np.array_equal(got, want)
    # the quantisation is visible: with the bf16 Q the cached keys' scores differ
    assert not np.allclose(got, oracle.cached_step(q, k, v, kc, vc, P, SCALE), atol=1e-6)
