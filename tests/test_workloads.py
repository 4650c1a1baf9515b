"""Workload shapes against the token arithmetic the pages print or imply
(tests/golden/token_arithmetic.txt, cited there)."""
import os

from block_causal_attention_dit_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "token_arithmetic.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        lines = f.readlines()
    for line in lines:
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def test_latent_grid_tokens():
    g = _golden()
    assert W.workload(1).requests[0].target == g["latent_tokens_1024"]
    assert W.workload(3).requests[0].target == g["latent_tokens_2048"]


def test_four_reference_target_share_is_about_a_fifth():
    g = _golden()
    r = W.workload(2).requests[0]
    assert r.seq_len == 20960
    share = r.target / r.seq_len
    assert g["four_ref_target_share_low"] <= share <= g["four_ref_target_share_high"]


def test_reference_token_counts():
    assert W.ref_tokens(1, 1) == 4096
    assert W.ref_tokens(9, 16) == 4080 and W.ref_tokens(16, 9) == 4080
    assert W.ref_tokens(3, 4) == 4070 and W.ref_tokens(4, 3) == 4070


def test_serving_batch_shape():
    wl = W.workload(4)
    assert len(wl.requests) == 8 and wl.kv_dtype == "fp8"
    for r in wl.requests:
        assert r.target == 4096
        assert 77 <= r.blocks[0] <= 1024
        assert 0 <= len(r.blocks) - 2 <= 4
        assert all(b in (4096, 4070, 4080) for b in r.blocks[1:-1])


def test_seeds_are_distinct():
    seen = set()
    for layer in range(32):
        for step in range(40):
            for req in range(8):
                for t in range(3):
                    seen.add(W.seed_for(4, layer, step, req, t))
    assert len(seen) == 32 * 40 * 8 * 3
