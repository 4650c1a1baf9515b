"""bca_step_attend_q8 on the GPU against the oracle's e4m3-Q reading of the cached
step on the same seeded inputs: each request's Q quantised per head with the
prefix cache's encoder ("Qwen/Qwen-Image-2.1" vLLM recipe, "Prefix KV cache",
applied to Q), the cached keys' scores taken from the e4m3 Q and e4m3 K, the own
keys' from the bf16 Q.  The Q codes and scales are bit-exact; outputs meet the
e4m3-cache tolerance (rel-L2 <= 2e-2) against the oracle reading the same bytes."""
import math

import numpy as np
import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200 import workloads as W
from block_causal_attention_dit_b200.workloads import randn_bf16
from _parity import REL_L2_FP8, assert_parity, sample_rows

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def make_request(T, P, H, seed, device, cap=None):
    q, k, v = (randn_bf16((T, H, 128), seed * 8 + t, device) for t in range(3))
    pk = randn_bf16((max(P, 1), H, 128), seed * 8 + 3, device)
    pv = randn_bf16((max(P, 1), H, 128), seed * 8 + 4, device)
    slot = bca.KVSlot(cap if cap is not None else max(P, 1), H, "fp8")
    slot.buffer.fill_(0xFF)  # NaN codes in every unused row: must never be read
    bca.kv_store(pk, pv, P, slot, epoch=seed + 1)
    return dict(q=q, k=k, v=v, slot=slot, T=T, P=P)


def oracle_for(req, rows=None):
    s = req["slot"]
    torch.cuda.synchronize()
    q = req["q"].cpu()
    return oracle.cached_step(q, req["k"], req["v"], s.k_view().cpu(), s.v_view().cpu(),
                              req["P"], SCALE, k_kind=oracle.KIND_E4M3,
                              v_kind=oracle.KIND_E4M3, k_scale=s.k_scale_view().cpu().numpy(),
                              v_scale=s.v_scale_view().cpu().numpy(), rows=rows,
                              q8=oracle.quantize_prefix(q, req["T"]))


def run_batch(reqs, H, device, workspace=None):
    q = torch.cat([r["q"] for r in reqs])
    k = torch.cat([r["k"] for r in reqs])
    v = torch.cat([r["v"] for r in reqs])
    o = torch.full_like(q, float("nan"))
    cu = np.concatenate([[0], np.cumsum([r["T"] for r in reqs])]).astype(np.int64)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    scratch = bca.step_attend_q8(q, k, v, o, cu, [r["slot"] for r in reqs], SCALE,
                                 workspace=workspace, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, cu, scratch


def test_q_codes_and_scales_are_the_cache_encoders(cuda_device):
    """The pre-pass's codes [H, rows, 128] and per-request scales equal the oracle's
    quantisation of each request's Q rows, byte for byte."""
    dev, H = cuda_device, 3
    reqs = [make_request(T, P, H, 40 + i, dev) for i, (T, P) in
            enumerate([(300, 129), (0, 40), (77, 1000), (256, 5)])]
    o, cu, scratch = run_batch(reqs, H, dev)
    codes, scales = bca.q8_views(scratch, int(cu[-1]), len(reqs), H)
    for i, r in enumerate(reqs):
        if r["T"] == 0:
            continue
        want_c, want_s = oracle.quantize_prefix(r["q"].cpu(), r["T"])
        assert np.array_equal(codes[:, cu[i]:cu[i + 1]].cpu().numpy(), want_c), f"request {i}"
        assert np.array_equal(scales[i].cpu().numpy(), want_s), f"request {i}"


@pytest.mark.parametrize("T,P,H", [(256, 128, 4), (300, 129, 2), (77, 1000, 2), (129, 0, 2),
                                   (1, 5, 1), (513, 640, 2), (128, 128, 1)])
def test_single_request(cuda_device, T, P, H):
    req = make_request(T, P, H, seed=5 * T + P, device=cuda_device, cap=P + 9)
    o, _, _ = run_batch([req], H, cuda_device)
    assert_parity(o, oracle_for(req), rel_l2=REL_L2_FP8, what=f"q8 T={T} P={P}")


@pytest.mark.parametrize("split", [False, True])
def test_ragged_batch(cuda_device, split):
    H = 2
    shapes = [(300, 513), (77, 0), (0, 20), (256, 1), (130, 2000), (1024, 2500)]
    reqs = [make_request(T, P, H, seed=500 + i, device=cuda_device, cap=P + 3)
            for i, (T, P) in enumerate(shapes)]
    ws = bca.step_workspace(cuda_device) if split else None
    o, cu, _ = run_batch(reqs, H, cuda_device, workspace=ws)
    for i, r in enumerate(reqs):
        if r["T"] == 0:
            continue
        assert_parity(o[cu[i]:cu[i + 1]], oracle_for(r), rel_l2=REL_L2_FP8, what=f"req {i}")


def test_serving_batch_sampled_rows(cuda_device):
    """The step-batched serving workload (8 requests, ragged prefixes of 77..~17k
    tokens, target 4096, H=32, e4m3 K and V cache) in the benchmark's launch
    configuration (workspace, split last round); sampled rows of every request."""
    wl = W.workload(4)
    dev = cuda_device
    slots, qs, ks_, vs_ = [], [], [], []
    for i, r in enumerate(wl.requests):
        q0, k0, v0 = W.qkv(wl, 0, 0, i, dev)
        slot = bca.KVSlot(r.prefix, wl.heads, "fp8")
        bca.prefill(q0, k0, v0, torch.empty_like(q0), r.offsets, wl.scale, slot=slot, epoch=1)
        slots.append(slot)
        del q0, k0, v0
        q, k, v = W.qkv(wl, 0, 1, i, dev)
        qs.append(q), ks_.append(k), vs_.append(v)
    q, k, v = torch.cat(qs), torch.cat(ks_), torch.cat(vs_)
    o = torch.empty_like(q)
    cu = np.concatenate([[0], np.cumsum([r.target for r in wl.requests])])
    bca.step_attend_q8(q, k, v, o, cu, slots, wl.scale, workspace=bca.step_workspace(dev))
    torch.cuda.synchronize()
    for i, r in enumerate(wl.requests):
        rows = sample_rows(r.target, 12, seed=i, boundaries=(128, 256, 2048))
        s = slots[i]
        qc = qs[i].cpu()
        want = oracle.cached_step(qc, ks_[i], vs_[i], s.k_view().cpu(), s.v_view().cpu(),
                                  r.prefix, wl.scale, k_kind=oracle.KIND_E4M3,
                                  v_kind=oracle.KIND_E4M3,
                                  k_scale=s.k_scale_view().cpu().numpy(),
                                  v_scale=s.v_scale_view().cpu().numpy(), rows=rows,
                                  q8=oracle.quantize_prefix(qc, r.target))
        got = o[cu[i]:cu[i + 1]][torch.from_numpy(rows).to(dev)]
        assert_parity(got, want, rel_l2=REL_L2_FP8, what=f"serving request {i}")


def test_repeated_batches_are_bitwise_identical(cuda_device):
    H = 4
    reqs = [make_request(T, P, H, seed=600 + i, device=cuda_device, cap=P)
            for i, (T, P) in enumerate([(512, 3000), (300, 129), (1024, 2500)])]
    first, _, _ = run_batch(reqs, H, cuda_device)
    for _ in range(3):
        again, _, _ = run_batch(reqs, H, cuda_device)
        assert torch.equal(first, again)


def test_argument_errors(cuda_device):
    H = 2
    fp8 = make_request(64, 32, H, 700, cuda_device)
    q, k, v = fp8["q"], fp8["k"], fp8["v"]
    o = torch.empty_like(q)
    bf16_slot = bca.KVSlot(32, H, "bf16")
    bca.kv_store(k[:32], v[:32], 32, bf16_slot, epoch=1)
    with pytest.raises(bca.BcaError) as e:
        bca.step_attend_q8(q, k, v, o, [0, 64], [bf16_slot], SCALE)
    assert e.value.status == 2  # e4m3 Q needs e4m3 K
    small = torch.empty(1024, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(bca.BcaError) as e:
        bca.step_attend_q8(q, k, v, o, [0, 64], [fp8["slot"]], SCALE, q8_scratch=small)
    assert e.value.status == 3
    o2, _, _ = run_batch([fp8], H, cuda_device)
    assert_parity(o2, oracle_for(fp8), rel_l2=REL_L2_FP8, what="after rejected calls")
