"""CUDA-graph replay of the cached step: capturing bca_step_attend (and a prefill +
cached steps sequence over several layers) and replaying it gives bit-identical
outputs to eager execution -- the property the pages report for CUDA graphs
("SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll": identical pixels with
graphs; "Qwen/Qwen-Image-2.1", "CUDA graphs": decode steps are captured)."""
import math

import pytest
import torch

import block_causal_attention_dit_b200 as bca
from block_causal_attention_dit_b200.workloads import randn_bf16

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def _warm(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_step_attend_graph_replay_is_bit_identical(cuda_device, mode):
    H, T, P = 32, 4096, 512  # split last round included
    q, k, v = (randn_bf16((T, H, 128), 500 + t, cuda_device) for t in range(3))
    pk, pv = (randn_bf16((P, H, 128), 510 + t, cuda_device) for t in range(2))
    slot = bca.KVSlot(P, H, mode)
    bca.kv_store(pk, pv, P, slot, epoch=1)
    ws = bca.step_workspace(cuda_device)
    o_eager, o_graph = torch.empty_like(q), torch.empty_like(q)
    call = lambda out: bca.step_attend(q, k, v, out, [0, T], [slot], SCALE, workspace=ws)
    _warm(lambda: call(o_graph))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(o_graph)
    for seed in (0, 1):
        if seed:  # new inputs in the same buffers, as a denoising loop would do
            for x, s in ((q, 520), (k, 521), (v, 522)):
                x.copy_(randn_bf16((T, H, 128), s, cuda_device))
        call(o_eager)
        o_graph.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o_graph, o_eager)


def test_prefill_and_steps_over_layers_graph_replay(cuda_device):
    """One graph holding prefill (with prefix store) and two cached steps for three
    layers, replayed twice, equals the eager sequence."""
    H, blocks = 8, [300, 700]
    S, P = sum(blocks), blocks[0]
    layers = []
    for l in range(3):
        qkv = tuple(randn_bf16((S, H, 128), 600 + 4 * l + t, cuda_device) for t in range(3))
        tgt = tuple(randn_bf16((blocks[1], H, 128), 700 + 4 * l + t, cuda_device) for t in range(3))
        layers.append((qkv, tgt, bca.KVSlot(P, H), torch.empty_like(qkv[0]),
                       torch.empty_like(tgt[0])))
    ws = bca.step_workspace(cuda_device)

    def run():
        for (q, k, v), (qt, kt, vt), slot, o, ot in layers:
            bca.prefill(q, k, v, o, [0, P, S], SCALE, slot=slot, epoch=1)
            for _ in range(2):
                bca.step_attend(qt, kt, vt, ot, [0, blocks[1]], [slot], SCALE, workspace=ws)

    _warm(run)
    eager = [(o.clone(), ot.clone()) for *_, o, ot in layers]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(2):
        for *_, o, ot in layers:
            o.zero_()
            ot.zero_()
        g.replay()
        torch.cuda.synchronize()
        for (a, b), (*_, o, ot) in zip(eager, layers):
            assert torch.equal(o, a) and torch.equal(ot, b)
