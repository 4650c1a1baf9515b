"""bca_step_graph: the cached-step attention of all layers of one layout recorded
once and replayed with one launch ("Qwen-Image-2.1 + vLLM-Omni day-0", "Serving
architecture: the cross-step prefix KV cache": CUDA graphs remove the step loop's
launch cost; "Qwen/Qwen-Image-2.1", "CUDA graphs": one captured entry per image
layout).  Replays read the activation buffers and cache slots in place, so new
contents between replays are used, and every replay is bit-identical to the eager
bca_step_attend calls on the same contents; the eager calls are themselves held to
the oracle by the step_attend parity tests, and one layer here is checked against
the oracle directly."""
import math

import numpy as np
import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200.workloads import randn_bf16
from tests._parity import assert_parity

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def _layout(device, H, targets, prefixes, layers, mode="bf16", seed=0):
    """Per layer: packed target q/k/v/o and one filled slot per request."""
    T = sum(targets)
    cu = [0]
    for t in targets:
        cu.append(cu[-1] + t)
    L = []
    for l in range(layers):
        q, k, v = (randn_bf16((T, H, 128), seed + 100 * l + t, device) for t in range(3))
        slots = []
        for r, P in enumerate(prefixes):
            pk, pv = (randn_bf16((max(P, 1), H, 128), seed + 100 * l + 10 + 2 * r + t, device)
                      for t in range(2))
            s = bca.KVSlot(max(P, 1), H, mode, device=device)
            bca.kv_store(pk, pv, P, s, epoch=1)
            slots.append((s, pk[:P], pv[:P]))
        L.append(dict(q=q, k=k, v=v, o=torch.empty_like(q), slots=slots))
    return cu, L


def _graph(cu, L, ws=None, status=None):
    return bca.StepGraph([x["q"] for x in L], [x["k"] for x in L], [x["v"] for x in L],
                         [x["o"] for x in L], cu, [[s for s, *_ in x["slots"]] for x in L],
                         SCALE, workspace=ws, dev_status=status)


def _eager(cu, L, ws=None):
    outs = []
    for x in L:
        o = torch.empty_like(x["q"])
        bca.step_attend(x["q"], x["k"], x["v"], o, cu, [s for s, *_ in x["slots"]], SCALE,
                        workspace=ws)
        outs.append(o)
    return outs


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_graph_replay_equals_eager_and_reads_buffers_in_place(cuda_device, mode):
    H = 4
    cu, L = _layout(cuda_device, H, [256, 131, 300], [128, 0, 77], layers=3, mode=mode)
    ws = bca.step_workspace(cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    g = _graph(cu, L, ws, status)
    assert g.kernel_nodes >= 3
    for rnd in range(3):
        if rnd:  # new contents in the same buffers, as the denoising loop writes them
            for l, x in enumerate(L):
                for j, name in enumerate("qkv"):
                    x[name].copy_(randn_bf16(tuple(x[name].shape), 9000 + 10 * rnd + 3 * l + j,
                                             cuda_device))
        for x in L:
            x["o"].fill_(float("nan"))
        g.launch()
        eager = _eager(cu, L, ws)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for x, e in zip(L, eager):
            assert torch.equal(x["o"], e)
    g.close()


def test_graph_layer_against_oracle(cuda_device):
    H = 4
    cu, L = _layout(cuda_device, H, [256, 100], [128, 40], layers=2, seed=50)
    g = _graph(cu, L)
    g.launch()
    torch.cuda.synchronize()
    x = L[1]
    o = x["o"].cpu()
    for r in range(2):
        s, pk, pv = x["slots"][r]
        sl = slice(cu[r], cu[r + 1])
        want = oracle.cached_step(x["q"][sl].cpu(), x["k"][sl].cpu(), x["v"][sl].cpu(),
                                  pk.cpu().permute(1, 0, 2).contiguous(),
                                  pv.cpu().permute(1, 0, 2).contiguous(), s.n_tokens, SCALE)
        assert_parity(o[sl], want, what=f"graph layer 1 request {r}")


def test_graph_with_split_schedule_many_replays(cuda_device):
    """T2I-shaped layer (4096 target rows, 512 cached keys, 32 heads): the schedule
    splits the last round, so each layer records the attention and the chunk-merge
    kernels; ten replays in a row all equal the eager result."""
    cu, L = _layout(cuda_device, 32, [4096], [512], layers=2, seed=70)
    ws = bca.step_workspace(cuda_device)
    g = _graph(cu, L, ws)
    assert g.kernel_nodes == 4
    eager = _eager(cu, L, ws)
    for _ in range(10):
        g.launch()
    torch.cuda.synchronize()
    for x, e in zip(L, eager):
        assert torch.equal(x["o"], e)


def test_graph_creation_reports_the_failing_layer(cuda_device):
    cu, L = _layout(cuda_device, 4, [256], [128], layers=3, seed=90)
    L[1]["slots"][0][0].struct.epoch = 0  # layer 1's slot was never filled
    with pytest.raises(bca.BcaError) as e:
        _graph(cu, L)
    assert e.value.status == 4
    L[1]["slots"][0][0].struct.epoch = 1
    g = _graph(cu, L)  # the library is usable afterwards
    g.launch()
    torch.cuda.synchronize()
    assert torch.equal(L[2]["o"], _eager(cu, L)[2])


def test_graph_without_target_rows_is_a_no_op(cuda_device):
    cu, L = _layout(cuda_device, 4, [0], [128], layers=2, seed=95)
    g = _graph(cu, L)
    assert g.kernel_nodes == 0
    g.launch()
    torch.cuda.synchronize()


def test_e4m3_q_graph_replay_equals_eager(cuda_device):
    """With a q8 scratch the graph records each layer's bca_step_attend_q8 (its Q
    quantisation kernels included): replays, also after new contents are written
    into the same buffers, are bit-identical to the eager e4m3-Q calls."""
    H = 4
    cu, L = _layout(cuda_device, H, [256, 131, 300], [128, 0, 77], layers=2, mode="fp8",
                    seed=70)
    ws = bca.step_workspace(cuda_device)
    scratch = bca.step_q8_scratch(cu[-1], len(cu) - 1, H, cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    g = bca.StepGraph([x["q"] for x in L], [x["k"] for x in L], [x["v"] for x in L],
                      [x["o"] for x in L], cu, [[s for s, *_ in x["slots"]] for x in L], SCALE,
                      workspace=ws, dev_status=status, q8_scratch=scratch)
    assert g.kernel_nodes >= 2 * 2  # per layer: the Q quantisation kernel + attention
    for rnd in range(2):
        if rnd:
            for l, x in enumerate(L):
                x["q"].copy_(randn_bf16(tuple(x["q"].shape), 9500 + l, cuda_device))
        g.launch()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for x in L:
            o = torch.empty_like(x["q"])
            bca.step_attend_q8(x["q"], x["k"], x["v"], o, cu, [s for s, *_ in x["slots"]],
                               SCALE, workspace=ws)
            torch.cuda.synchronize()
            assert torch.equal(x["o"], o)
    g.close()


def test_dq_graph_replay_equals_eager(cuda_device):
    """With a dq scratch the graph records each layer's bca_step_attend_dq (its
    expansion kernel included): replays, also after new contents are written into the
    same buffers, are bit-identical to the eager dq calls and to bca_step_attend."""
    H = 4
    cu, L = _layout(cuda_device, H, [256, 131, 300], [128, 0, 77], layers=2, mode="fp8",
                    seed=90)
    ws = bca.step_workspace(cuda_device)
    scratch = torch.empty(max(bca.step_dq_scratch_bytes([s for s, *_ in x["slots"]])
                              for x in L), dtype=torch.uint8, device=cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    g = bca.StepGraph([x["q"] for x in L], [x["k"] for x in L], [x["v"] for x in L],
                      [x["o"] for x in L], cu, [[s for s, *_ in x["slots"]] for x in L], SCALE,
                      workspace=ws, dev_status=status, dq_scratch=scratch)
    assert g.kernel_nodes >= 2 * 2  # per layer: the expansion kernel + attention
    for rnd in range(2):
        if rnd:
            for l, x in enumerate(L):
                x["q"].copy_(randn_bf16(tuple(x["q"].shape), 9600 + l, cuda_device))
        g.launch()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for x in L:
            slots = [s for s, *_ in x["slots"]]
            o, o2 = torch.empty_like(x["q"]), torch.empty_like(x["q"])
            bca.step_attend_dq(x["q"], x["k"], x["v"], o, cu, slots, SCALE, workspace=ws)
            bca.step_attend(x["q"], x["k"], x["v"], o2, cu, slots, SCALE, workspace=ws)
            torch.cuda.synchronize()
            assert torch.equal(x["o"], o) and torch.equal(o, o2)
    g.close()
    with pytest.raises(bca.BcaError):
        bca.StepGraph([x["q"] for x in L], [x["k"] for x in L], [x["v"] for x in L],
                      [x["o"] for x in L], cu, [[s for s, *_ in x["slots"]] for x in L], SCALE,
                      q8_scratch=scratch, dq_scratch=scratch)
