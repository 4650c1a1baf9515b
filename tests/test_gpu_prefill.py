"""bca_prefill on the GPU against the oracle: block-causal attention over the whole
sequence ("Qwen-Image-2.1 + vLLM-Omni day-0", "What is Qwen-Image-2.1": block b
attends to blocks 0..b, full attention inside a block) and the prefix K/V it
stores for later steps ("Serving architecture: the cross-step prefix KV cache")."""
import math

import numpy as np
import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200 import workloads as W
from block_causal_attention_dit_b200.workloads import randn_bf16
from _parity import assert_parity, sample_rows

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def offsets(blocks):
    return [0] + np.cumsum(blocks).tolist()


def run(blocks, H, seed, device, slot=None, epoch=0):
    S = int(sum(blocks))
    q, k, v = (randn_bf16((S, H, 128), seed * 4 + t, device) for t in range(3))
    o = torch.full_like(q, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=device)
    bca.prefill(q, k, v, o, offsets(blocks), SCALE, slot=slot, epoch=epoch, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return q, k, v, o


@pytest.mark.parametrize("blocks,H", [
    ([128, 256], 4),            # the tiny workload's shape
    ([77, 130, 300], 2),        # boundaries off the 128 grid
    ([384], 2),                 # a single block: plain full attention
    ([1, 1, 1, 256], 1),        # unit blocks at the start
    ([5] * 40 + [100], 2),      # many small blocks inside one tile
    ([300, 1], 3),              # a one-token target
    ([1], 1),
    ([129, 127, 2, 255], 2),
])
def test_prefill_all_rows(cuda_device, blocks, H):
    q, k, v, o = run(blocks, H, seed=sum(blocks) + len(blocks), device=cuda_device)
    want = oracle.prefill(q, k, v, offsets(blocks), SCALE)
    assert_parity(o, want, what=str(blocks))


def test_prefill_stores_prefix_and_cached_step_matches(cuda_device):
    """The slot receives the exact prefix K/V; a cached step on the target rows with
    that slot reproduces the prefill's target rows (both against the oracle)."""
    blocks, H = [200, 130, 333], 2
    P = sum(blocks[:-1])
    slot = bca.KVSlot(P + 10, H)
    q, k, v, o = run(blocks, H, 77, cuda_device, slot=slot, epoch=9)
    assert slot.n_tokens == P and slot.epoch == 9
    assert torch.equal(slot.k_view()[:, :P], k[:P].permute(1, 0, 2))
    assert torch.equal(slot.v_view()[:, :P], v[:P].permute(1, 0, 2))
    want = oracle.prefill(q, k, v, offsets(blocks), SCALE)
    assert_parity(o, want)
    o2 = torch.empty_like(q[P:])
    bca.step_attend(q[P:], k[P:], v[P:], o2, [0, blocks[-1]], [slot], SCALE)
    torch.cuda.synchronize()
    assert_parity(o2, want[P:], what="cached step vs recompute")


def test_prefix_outputs_ignore_the_target(cuda_device):
    blocks, H = [150, 300, 200], 2
    P = sum(blocks[:-1])
    q, k, v, o = run(blocks, H, 5, cuda_device)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    for x in (q2, k2, v2):
        x[P:] = randn_bf16(tuple(x[P:].shape), 999, cuda_device) * 4
    o2 = torch.empty_like(q)
    bca.prefill(q2, k2, v2, o2, offsets(blocks), SCALE)
    torch.cuda.synchronize()
    assert torch.equal(o[:P], o2[:P])


@pytest.mark.parametrize("ws", [False, True])
@pytest.mark.parametrize("wl_index", [1, 2, 3])
def test_full_size_sampled_rows(cuda_device, wl_index, ws):
    """The T2I, 4-ref edit and native-2K shapes (H=32) at one layer, sampled rows x
    all heads, including every block boundary +-1; with a workspace (the benchmark's
    configuration: heavy pairs' last round split) and without."""
    wl = W.workload(wl_index)
    req = wl.requests[0]
    q, k, v = W.qkv(wl, 0, 0, 0, cuda_device)
    o = torch.empty_like(q)
    bca.prefill(q, k, v, o, req.offsets, wl.scale,
                workspace=bca.step_workspace(cuda_device) if ws else None)
    torch.cuda.synchronize()
    rows = sample_rows(req.seq_len, 48, seed=wl_index, boundaries=req.offsets[1:-1])
    want = oracle.prefill(q, k, v, req.offsets, wl.scale, rows=rows)
    assert_parity(o[torch.from_numpy(rows).to(cuda_device)], want, what=wl.name)


def test_many_items_per_cta_with_half_empty_q_pairs(cuda_device):
    """S = 384: the second pair of every head has one 128-row tile and an empty one;
    H = 256 gives 512 work items, several per CTA, so Q buffers are reused across
    items that have an absent tile."""
    blocks, H = [100, 284], 256
    q, k, v, o = run(blocks, H, 31, cuda_device)
    rows = sample_rows(384, 48, seed=5, boundaries=(100, 128, 256))
    want = oracle.prefill(q, k, v, offsets(blocks), SCALE, rows=rows)
    assert_parity(o[torch.from_numpy(rows).to(cuda_device)], want, what="half-empty pairs")


@pytest.mark.parametrize("blocks,H", [
    ([300, 200, 1500], 8),      # a split pair straddles two block ends
    ([128, 256], 4),            # the tiny workload
    ([512, 4096], 2),           # T2I blocks, few heads: every heavy pair split
    ([77, 130, 300, 2000], 6),
])
def test_prefill_with_workspace_all_rows(cuda_device, blocks, H):
    """bca_prefill_ws: heavy Q-tile pairs first, the last partial round of them split
    along the keys, light pairs after.  A split chunk may hold rows whose block ends
    before the chunk's keys begin (their chunk is empty), or a whole Q tile with no
    key in the chunk; all rows against the oracle."""
    S = int(sum(blocks))
    q, k, v = (randn_bf16((S, H, 128), 4000 + S + t, cuda_device) for t in range(3))
    o = torch.full_like(q, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bca.prefill(q, k, v, o, offsets(blocks), SCALE, dev_status=status,
                workspace=bca.step_workspace(cuda_device))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_parity(o, oracle.prefill(q, k, v, offsets(blocks), SCALE), what=f"ws {blocks}")
