"""Seeded synthetic workloads shaped like the pages' generation requests.

This module holds shapes and random numbers only (none of the method's
arithmetic), so both the CUDA path's tests/benchmark and the oracle can be fed
from it.

Shapes (cited by page title and section):
  * 1024x1024 text-to-image, 40 steps, CFG off -- "Qwen/Qwen-Image-2.1" (vLLM
    recipe), "Sampling defaults"; B200 latency quoted for that shape on
    "SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll" (orcarouter.ai).
  * The autoencoder compresses 16x, so a 1024^2 image is a 64x64 = 4096-token
    latent grid and 2048^2 is 128x128 = 16384 tokens -- recipe, component table.
  * Up to 4 reference images, each resized to ~1024x1024 of area with its own
    aspect ratio -- recipe, "Offline inference".
  * --step-execution --max-num-seqs 8 batches requests at the same KV-cache
    phase -- recipe, "Online serving".
  * DiT: 32 layers -- "Qwen-Image-2.1: SGLang vs vLLM-Omni Measured on a Single
    L20", introduction.  H = 32 heads of head_dim 128 is a reading (the pages give no
    head count).

Inputs: bf16 <- fp32 N(0, 1) from torch.randn with a seeded torch.Generator on
the target device, rounded to bf16 (RNE).  Seed of tensor t (q=0, k=1, v=2) of
request r at (layer, step) of workload c: (((c*100 + layer)*100 + step)*16 + r)*4 + t.
Step 0 is the prefill (whole sequence); steps >= 1 draw fresh target rows.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128
# Aspect ratios (height:width) a reference image may take.
REF_ASPECTS = ((1, 1), (3, 4), (4, 3), (9, 16), (16, 9))


def ref_tokens(h_ratio: int, w_ratio: int, area_tokens: int = 4096) -> int:
    """Latent tokens of one reference image resized to ~area_tokens of area:
    h = round(sqrt(area * h/w)), w = floor(area / h); 1:1 -> 4096, 3:4 -> 4070,
    9:16 -> 4080."""
    h = int(round(math.sqrt(area_tokens * h_ratio / w_ratio)))
    w = area_tokens // h
    return h * w


@dataclass
class Request:
    """One generation request: ordered blocks (text, refs..., target)."""
    blocks: list  # token counts; the last block is the target

    @property
    def prefix(self) -> int:
        return int(sum(self.blocks[:-1]))

    @property
    def target(self) -> int:
        return int(self.blocks[-1])

    @property
    def seq_len(self) -> int:
        return int(sum(self.blocks))

    @property
    def offsets(self) -> list:
        off = [0]
        for b in self.blocks:
            off.append(off[-1] + int(b))
        return off


@dataclass
class Workload:
    index: int
    name: str
    heads: int
    requests: list
    layers: int
    steps: int
    kv_dtype: str = "bf16"  # "bf16" | "fp8_v" | "fp8"
    head_dim: int = HEAD_DIM
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


def sample_serving_requests(n_requests: int = 8, seed: int = 4) -> list:
    """Ragged same-phase batch: text ~ U{77..1024}, 0..4 refs, each ref's aspect
    uniform over REF_ASPECTS, target 4096 tokens (64x64)."""
    rng = np.random.default_rng(seed)
    reqs = []
    for _ in range(n_requests):
        text = int(rng.integers(77, 1025))
        n_refs = int(rng.integers(0, 5))
        refs = [ref_tokens(*REF_ASPECTS[int(rng.integers(0, len(REF_ASPECTS)))])
                for _ in range(n_refs)]
        reqs.append(Request([text] + refs + [4096]))
    return reqs


def workload(index: int) -> Workload:
    if index == 0:
        return Workload(0, "tiny: H=4, blocks [text 128, target 256 (16x16)]", 4,
                        [Request([128, 256])], layers=1, steps=2)
    if index == 1:
        return Workload(1, "t2i 1024x1024: H=32, blocks [text 512, target 4096 (64x64)]", 32,
                        [Request([512, 4096])], layers=32, steps=40)
    if index == 2:
        return Workload(2, "4-ref edit: H=32, blocks [text 512, refs 4096/4080/4080/4096, "
                           "target 4096]", 32,
                        [Request([512, 4096, 4080, 4080, 4096, 4096])], layers=32, steps=40)
    if index == 3:
        return Workload(3, "native 2K: H=32, blocks [text 1024, ref 4096, target 16384 "
                           "(128x128)]", 32,
                        [Request([1024, 4096, 16384])], layers=32, steps=40)
    if index == 4:
        return Workload(4, "step-batched serving: 8 requests, ragged prefixes, target 4096, "
                           "fp8 (K and V) prefix cache", 32,
                        sample_serving_requests(), layers=32, steps=40, kv_dtype="fp8")
    raise ValueError(f"no workload {index}")


def seed_for(workload_index: int, layer: int, step: int, request: int, tensor: int) -> int:
    return (((workload_index * 100 + layer) * 100 + step) * 16 + request) * 4 + tensor


def randn_bf16(shape, seed: int, device="cpu"):
    """bf16 <- fp32 N(0,1), seeded, generated on `device`."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(
        torch.bfloat16)


def qkv(wl: Workload, layer: int, step: int, request: int, device="cpu"):
    """(q, k, v) for one request: step 0 -> the whole sequence [S, H, d];
    step >= 1 -> fresh target rows [T, H, d]."""
    req = wl.requests[request]
    rows = req.seq_len if step == 0 else req.target
    shape = (rows, wl.heads, wl.head_dim)
    return tuple(randn_bf16(shape, seed_for(wl.index, layer, step, request, t), device)
                 for t in range(3))
