"""bca_step_attend_q8 on the GPU against the oracle's e4m3-Q reading of the cached
step on the same seeded inputs: each request's Q quantised per head with the
prefix cache's encoder ("Qwen/Qwen-Image-2.1" vLLM recipe, "Prefix KV cache",
applied to Q), the cached keys' scores taken from the e4m3 Q and e4m3 K, the own
keys' from the bf16 Q.  The Q codes and scales are bit-exact.  The oracle models
the Q rounding exactly, so what is left between kernel and oracle is the kernel's
own bf16-P / fp32-sum error, as in the bf16 cached step: outputs are held to the
bf16 tolerance (max-abs <= 2e-2, rel-L2 <= 5e-3) against the e4m3-Q oracle.  Where
the e4m3-Q oracle and the plain (bf16-Q) oracle differ by more than twice that
tolerance, the kernel must also be strictly closer to the e4m3-Q one, so a kernel
that fed the bf16 Q (or another Q scale) to the cached keys fails; the shapes with
many cached keys are there to make that gap large, and the test asserts that it
is."""
import math

import numpy as np
import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200 import workloads as W
from block_causal_attention_dit_b200.workloads import randn_bf16
from _parity import REL_L2, assert_parity, errors, sample_rows, to_f64

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


def oracle_for(req, rows=None, q8=True):
    """The oracle over the slot's e4m3 bytes; q8=True: the e4m3-Q reading (Q codes
    from the oracle's own encoder), q8=False: the plain cached step (bf16 Q)."""
    s = req["slot"]
    torch.cuda.synchronize()
    q = req["q"].cpu()
    return oracle.cached_step(q, req["k"], req["v"], s.k_view().cpu(), s.v_view().cpu(),
                              req["P"], SCALE, k_kind=oracle.KIND_E4M3,
                              v_kind=oracle.KIND_E4M3, k_scale=s.k_scale_view().cpu().numpy(),
                              v_scale=s.v_scale_view().cpu().numpy(), rows=rows,
                              q8=oracle.quantize_prefix(q, req["T"]) if q8 else None)


def assert_q8(got, want_q8, want_plain, what="", must_discriminate=False):
    """got within the bf16 tolerance of the e4m3-Q oracle; where the two oracles are
    further apart than twice the tolerance, got must be closer to the e4m3-Q one.
    Returns the gap between the oracles (rel-L2)."""
    g = to_f64(got) if isinstance(got, torch.Tensor) else got
    assert_parity(g, want_q8, what=what)
    _, gap = errors(want_plain, want_q8)
    if must_discriminate:
        assert gap > 2 * REL_L2, f"{what}: oracles only {gap:.3e} apart"
    if gap > 2 * REL_L2:
        _, e_q8 = errors(g, want_q8)
        _, e_plain = errors(g, want_plain)
        assert e_q8 < e_plain, f"{what}: {e_q8:.3e} to the e4m3-Q oracle, {e_plain:.3e} to bf16-Q"
    return gap


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


# (T, P, H, must the two oracles be > 2x the tolerance apart?)  Shapes with P >= T
# are the ones where the Q rounding moves O by well over the tolerance; P = 0 and
# tiny P cover the edges (no or few cached keys: nothing to tell apart).
@pytest.mark.parametrize("T,P,H,disc", [(256, 128, 4, False), (300, 129, 2, False),
                                        (77, 1000, 2, True), (129, 0, 2, False),
                                        (1, 5, 1, False), (513, 640, 2, True),
                                        (128, 128, 1, False), (256, 1024, 2, True),
                                        (128, 2048, 1, True)])
def test_single_request(cuda_device, T, P, H, disc):
    req = make_request(T, P, H, seed=5 * T + P, device=cuda_device, cap=P + 9)
    o, _, _ = run_batch([req], H, cuda_device)
    assert_q8(o, oracle_for(req), oracle_for(req, q8=False), what=f"q8 T={T} P={P}",
              must_discriminate=disc)


@pytest.mark.parametrize("split", [False, True])
def test_ragged_batch(cuda_device, split):
    H = 2
    shapes = [(300, 513), (77, 0), (0, 20), (256, 1), (130, 2000), (1024, 2500)]
    reqs = [make_request(T, P, H, seed=500 + i, device=cuda_device, cap=P + 3)
            for i, (T, P) in enumerate(shapes)]
    ws = bca.step_workspace(cuda_device) if split else None
    o, cu, _ = run_batch(reqs, H, cuda_device, workspace=ws)
    gaps = []
    for i, r in enumerate(reqs):
        if r["T"] == 0:
            continue
        gaps.append(assert_q8(o[cu[i]:cu[i + 1]], oracle_for(r), oracle_for(r, q8=False),
                              what=f"req {i}"))
    assert max(gaps) > 2 * REL_L2  # at least one request tells the two readings apart


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
        want_plain = oracle.cached_step(qc, ks_[i], vs_[i], s.k_view().cpu(), s.v_view().cpu(),
                                        r.prefix, wl.scale, k_kind=oracle.KIND_E4M3,
                                        v_kind=oracle.KIND_E4M3,
                                        k_scale=s.k_scale_view().cpu().numpy(),
                                        v_scale=s.v_scale_view().cpu().numpy(), rows=rows)
        got = o[cu[i]:cu[i + 1]][torch.from_numpy(rows).to(dev)]
        # requests with at least as many cached keys as target rows must tell the
        # e4m3-Q reading from the bf16-Q one
        assert_q8(got, want, want_plain, what=f"serving request {i}",
                  must_discriminate=r.prefix >= r.target)


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
    assert_q8(o2, oracle_for(fp8), oracle_for(fp8, q8=False), what="after rejected calls")
