"""bca_step_attend on the GPU against the oracle on the same seeded inputs.
Target rows attend to [cached prefix ; own target K/V] ("Qwen-Image-2.1 +
vLLM-Omni day-0", "Serving architecture: the cross-step prefix KV cache";
same-phase batching: "Qwen/Qwen-Image-2.1" vLLM recipe, "Online serving")."""
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


def make_request(T, P, H, seed, device, cap=None, mode="bf16"):
    q, k, v = (randn_bf16((T, H, 128), seed * 8 + t, device) for t in range(3))
    pk = randn_bf16((max(P, 1), H, 128), seed * 8 + 3, device)
    pv = randn_bf16((max(P, 1), H, 128), seed * 8 + 4, device)
    slot = bca.KVSlot(cap if cap is not None else max(P, 1), H, mode)
    slot.buffer.fill_(0xFF)  # NaN patterns in every unused row: must never be read
    bca.kv_store(pk, pv, P, slot, epoch=seed + 1)
    return dict(q=q, k=k, v=v, pk=pk, pv=pv, slot=slot, T=T, P=P)


def oracle_for(req, rows=None):
    """The oracle's cached step for a request made by make_request.  A bf16 cache is
    built on the host from the source prefix rows (the slot's bytes are never read,
    so a store bug cannot cancel a matching read bug); an e4m3 cache is read from the
    slot, as the e4m3 rule compares against the same bytes (their equality with the
    oracle's own encoding is checked by the kv_store tests)."""
    s = req["slot"]
    torch.cuda.synchronize()
    if s.dtype == bca.KV_BF16:
        kc = req["pk"].cpu().permute(1, 0, 2).contiguous()
        vc = req["pv"].cpu().permute(1, 0, 2).contiguous()
        return oracle.cached_step(req["q"], req["k"], req["v"], kc, vc, req["P"], SCALE,
                                  rows=rows)
    kk = oracle.KIND_E4M3 if s.dtype == bca.KV_FP8_KV else oracle.KIND_BF16
    if kk == oracle.KIND_E4M3:
        kc = s.k_view().cpu()
    else:  # "fp8_v": bf16 K from the host rows, padded to the slot's capacity
        H, cap, P = s.struct.num_heads, s.struct.cap_tokens, req["P"]
        kc = torch.zeros((H, cap, 128), dtype=torch.bfloat16)
        kc[:, :P] = req["pk"][:P].cpu().permute(1, 0, 2)
    return oracle.cached_step(req["q"], req["k"], req["v"], kc, s.v_view().cpu(), req["P"],
                              SCALE, k_kind=kk, v_kind=oracle.KIND_E4M3,
                              k_scale=s.k_scale_view().cpu().numpy(),
                              v_scale=s.v_scale_view().cpu().numpy(), rows=rows)


def run_batch(reqs, H, device, workspace=None):
    q = torch.cat([r["q"] for r in reqs])
    k = torch.cat([r["k"] for r in reqs])
    v = torch.cat([r["v"] for r in reqs])
    o = torch.full_like(q, float("nan"))
    cu = np.concatenate([[0], np.cumsum([r["T"] for r in reqs])])
    status = torch.zeros(1, dtype=torch.int32, device=device)
    bca.step_attend(q, k, v, o, cu, [r["slot"] for r in reqs], SCALE, workspace=workspace,
                    dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, cu


@pytest.mark.parametrize("T,P,H", [(256, 128, 4), (77, 1, 2), (1, 0, 1), (300, 129, 2),
                                   (129, 255, 3), (513, 640, 2), (128, 128, 1), (255, 1000, 2)])
def test_single_request(cuda_device, T, P, H):
    req = make_request(T, P, H, seed=T + P, device=cuda_device, cap=P + 37)
    o, _ = run_batch([req], H, cuda_device)
    assert_parity(o, oracle_for(req), what=f"T={T} P={P}")


def test_tiny_workload_step_two(cuda_device):
    """The tiny workload: blocks [text 128, target 256], H=4; step 2 reuses the
    text K/V stored at step 1."""
    wl = W.workload(0)
    q0, k0, v0 = W.qkv(wl, 0, 0, 0, cuda_device)
    P = wl.requests[0].prefix
    slot = bca.KVSlot(P, wl.heads)
    bca.kv_store(k0, v0, P, slot, epoch=1)
    q, k, v = W.qkv(wl, 0, 1, 0, cuda_device)
    o = torch.empty_like(q)
    bca.step_attend(q, k, v, o, [0, q.shape[0]], [slot], wl.scale)
    torch.cuda.synchronize()
    kc = k0[:P].permute(1, 0, 2).contiguous()
    vc = v0[:P].permute(1, 0, 2).contiguous()
    want = oracle.cached_step(q, k, v, kc, vc, P, wl.scale)
    assert_parity(o, want, what="tiny step 2")


def test_ragged_batch(cuda_device):
    H = 2
    shapes = [(77, 0), (300, 200), (128, 513), (1, 7), (640, 129)]
    reqs = [make_request(T, P, H, seed=100 + i, device=cuda_device, cap=P + 5)
            for i, (T, P) in enumerate(shapes)]
    o, cu = run_batch(reqs, H, cuda_device)
    for i, r in enumerate(reqs):
        assert_parity(o[cu[i]:cu[i + 1]], oracle_for(r), what=f"request {i}")


def test_batch_with_empty_request(cuda_device):
    H = 2
    reqs = [make_request(130, 60, H, 7, cuda_device), make_request(0, 30, H, 8, cuda_device),
            make_request(90, 300, H, 9, cuda_device)]
    reqs[1]["q"] = reqs[1]["k"] = reqs[1]["v"] = torch.empty((0, H, 128), dtype=torch.bfloat16,
                                                              device=cuda_device)
    o, cu = run_batch(reqs, H, cuda_device)
    assert_parity(o[cu[0]:cu[1]], oracle_for(reqs[0]))
    assert_parity(o[cu[2]:cu[3]], oracle_for(reqs[2]))


def test_t2i_1024_sampled_rows(cuda_device):
    """Full-size text-to-image shape (H=32, text 512, target 4096) at one layer/step,
    checked on sampled target rows x all heads (plus tile boundaries)."""
    wl = W.workload(1)
    q0, k0, v0 = W.qkv(wl, 3, 0, 0, cuda_device)
    P = wl.requests[0].prefix
    slot = bca.KVSlot(P, wl.heads)
    bca.kv_store(k0, v0, P, slot, epoch=1)
    q, k, v = W.qkv(wl, 3, 5, 0, cuda_device)
    o = torch.empty_like(q)
    bca.step_attend(q, k, v, o, [0, q.shape[0]], [slot], wl.scale)
    torch.cuda.synchronize()
    rows = sample_rows(q.shape[0], 192, seed=1, boundaries=range(128, 4096, 128))
    kc = k0[:P].permute(1, 0, 2).contiguous()
    vc = v0[:P].permute(1, 0, 2).contiguous()
    want = oracle.cached_step(q, k, v, kc, vc, P, wl.scale, rows=rows)
    assert_parity(o[torch.from_numpy(rows).to(cuda_device)], want, what="t2i sampled")


@pytest.mark.parametrize("wl_index", [2, 3])
def test_full_size_cached_step_sampled_rows(cuda_device, wl_index):
    """The 4-ref edit (text 512 + four refs, target 4096: 16864 cached keys) and
    native-2K (text 1024 + ref 4096, target 16384) cached steps at full size, in the
    benchmark's launch configuration (workspace, split last round), sampled target
    rows x all heads plus KV-tile boundaries of the target +-1 (16 of them)."""
    wl = W.workload(wl_index)
    req = wl.requests[0]
    P = req.prefix
    q0, k0, v0 = W.qkv(wl, 2, 0, 0, cuda_device)
    slot = bca.KVSlot(P, wl.heads)
    bca.kv_store(k0, v0, P, slot, epoch=1)
    q, k, v = W.qkv(wl, 2, 7, 0, cuda_device)
    o = torch.empty_like(q)
    ws = bca.step_workspace(cuda_device)
    bca.step_attend(q, k, v, o, [0, q.shape[0]], [slot], wl.scale, workspace=ws)
    torch.cuda.synchronize()
    T = q.shape[0]
    tiles = list(range(128, T, 128))
    rows = sample_rows(T, 24, seed=10 + wl_index, boundaries=tiles[:: max(1, len(tiles) // 16)])
    kc = k0[:P].permute(1, 0, 2).contiguous()
    vc = v0[:P].permute(1, 0, 2).contiguous()
    want = oracle.cached_step(q, k, v, kc, vc, P, wl.scale, rows=rows)
    assert_parity(o[torch.from_numpy(rows).to(cuda_device)], want, what=f"{wl.name} cached step")


def test_repeated_calls_are_deterministic(cuda_device):
    req = make_request(300, 200, 2, 55, cuda_device)
    a, _ = run_batch([req], 2, cuda_device)
    b, _ = run_batch([req], 2, cuda_device)
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# e4m3 prefix cache ("Prefix KV cache": "fp8_v" quantises V, "fp8" K and V).
# Compared with the oracle reading the same cache bytes: rel-L2 <= 2e-2.
# ---------------------------------------------------------------------------
from _parity import REL_L2_FP8  # noqa: E402


@pytest.mark.parametrize("mode", ["fp8", "fp8_v"])
@pytest.mark.parametrize("T,P,H", [(256, 128, 4), (300, 129, 2), (77, 1000, 2), (129, 0, 2),
                                   (1, 5, 1)])
def test_fp8_cache_single_request(cuda_device, mode, T, P, H):
    req = make_request(T, P, H, seed=3 * T + P, device=cuda_device, cap=P + 11, mode=mode)
    o, _ = run_batch([req], H, cuda_device)
    assert_parity(o, oracle_for(req), rel_l2=REL_L2_FP8, what=f"{mode} T={T} P={P}")


@pytest.mark.parametrize("mode", ["fp8", "fp8_v"])
def test_fp8_cache_ragged_batch(cuda_device, mode):
    H = 2
    shapes = [(300, 513), (77, 0), (256, 1), (130, 2000)]
    reqs = [make_request(T, P, H, seed=200 + i, device=cuda_device, cap=P + 3, mode=mode)
            for i, (T, P) in enumerate(shapes)]
    o, cu = run_batch(reqs, H, cuda_device)
    for i, r in enumerate(reqs):
        assert_parity(o[cu[i]:cu[i + 1]], oracle_for(r), rel_l2=REL_L2_FP8, what=f"req {i}")


def test_prefill_into_fp8_slot_then_cached_step(cuda_device):
    H, blocks = 2, [100, 333, 200]
    S, P = sum(blocks), sum(blocks[:-1])
    q, k, v = (randn_bf16((S, H, 128), 300 + t, cuda_device) for t in range(3))
    o = torch.empty_like(q)
    slot = bca.KVSlot(P, H, "fp8")
    bca.prefill(q, k, v, o, [0, 100, 433, S], SCALE, slot=slot, epoch=4)
    torch.cuda.synchronize()
    kc, ks = oracle.quantize_prefix(k.cpu(), P)
    vc, vs = oracle.quantize_prefix(v.cpu(), P)
    assert np.array_equal(slot.k_view().cpu().numpy(), kc)
    assert np.array_equal(slot.v_view().cpu().numpy(), vc)
    assert np.array_equal(slot.k_scale_view().cpu().numpy(), ks)
    assert np.array_equal(slot.v_scale_view().cpu().numpy(), vs)
    qt, kt, vt = q[P:], k[P:], v[P:]
    ot = torch.empty_like(qt)
    bca.step_attend(qt, kt, vt, ot, [0, S - P], [slot], SCALE)
    torch.cuda.synchronize()
    want = oracle.cached_step(qt, kt, vt, kc, vc, P, SCALE, k_kind=oracle.KIND_E4M3,
                              v_kind=oracle.KIND_E4M3, k_scale=ks, v_scale=vs)
    assert_parity(ot, want, rel_l2=REL_L2_FP8, what="fp8 slot from prefill")


def test_serving_batch_sampled_rows(cuda_device):
    """The step-batched serving workload: 8 requests with ragged prefixes (77..~17k
    tokens), target 4096 each, H=32, e4m3 K and V cache; sampled target rows of
    every request x all heads."""
    wl = W.workload(4)
    slots, qs, ks_, vs_ = [], [], [], []
    for i, r in enumerate(wl.requests):
        q0, k0, v0 = W.qkv(wl, 0, 0, i, cuda_device)
        slot = bca.KVSlot(r.prefix, wl.heads, "fp8")
        bca.prefill(q0, k0, v0, torch.empty_like(q0), r.offsets, wl.scale, slot=slot, epoch=1)
        slots.append(slot)
        del q0, k0, v0
        q, k, v = W.qkv(wl, 0, 1, i, cuda_device)
        qs.append(q), ks_.append(k), vs_.append(v)
    q, k, v = torch.cat(qs), torch.cat(ks_), torch.cat(vs_)
    o = torch.empty_like(q)
    cu = np.concatenate([[0], np.cumsum([r.target for r in wl.requests])])
    bca.step_attend(q, k, v, o, cu, slots, wl.scale)
    torch.cuda.synchronize()
    for i, r in enumerate(wl.requests):
        rows = sample_rows(r.target, 12, seed=i, boundaries=(128, 256, 2048))
        s = slots[i]
        want = oracle.cached_step(qs[i], ks_[i], vs_[i], s.k_view().cpu(), s.v_view().cpu(),
                                  r.prefix, wl.scale, k_kind=oracle.KIND_E4M3,
                                  v_kind=oracle.KIND_E4M3,
                                  k_scale=s.k_scale_view().cpu().numpy(),
                                  v_scale=s.v_scale_view().cpu().numpy(), rows=rows)
        got = o[cu[i]:cu[i + 1]][torch.from_numpy(rows).to(cuda_device)]
        assert_parity(got, want, rel_l2=REL_L2_FP8, what=f"serving request {i}")


@pytest.mark.parametrize("mode", ["fp8", "fp8_v", "bf16"])
def test_repeated_batches_are_bitwise_identical(cuda_device, mode):
    """Races between the producer, converter, MMA and softmax roles would show up as
    run-to-run differences; the kernel is deterministic, so outputs must repeat."""
    H = 4
    shapes = [(512, 3000), (300, 129), (1024, 2500)]
    reqs = [make_request(T, P, H, seed=400 + i, device=cuda_device, cap=P, mode=mode)
            for i, (T, P) in enumerate(shapes)]
    first, _ = run_batch(reqs, H, cuda_device)
    for _ in range(4):
        again, _ = run_batch(reqs, H, cuda_device)
        assert torch.equal(first, again)


# ---------------------------------------------------------------------------
# Split last round: with a workspace, units of the last partial round are split
# along the keys and merged by a second kernel.
# ---------------------------------------------------------------------------
def test_split_tail_matches_oracle_and_unsplit(cuda_device):
    """H=32, T=4096, P=512 gives 512 units on 148 SMs: 68 leftover units are split."""
    H = 32
    req = make_request(4096, 512, H, seed=900, device=cuda_device)
    ws = bca.step_workspace(cuda_device)
    assert bca.step_workspace_bytes() > 0
    a, _ = run_batch([req], H, cuda_device, workspace=ws)
    b, _ = run_batch([req], H, cuda_device)
    rows = sample_rows(4096, 160, seed=9, boundaries=range(256, 4096, 256))
    want = oracle_for(req, rows=rows)
    idx = torch.from_numpy(rows).to(cuda_device)
    assert_parity(a[idx], want, what="split")
    assert_parity(b[idx], want, what="unsplit")
    # the unsplit rows of both runs are computed identically
    diff = (a.float() - b.float()).abs().amax(dim=(1, 2))
    assert float(diff.max()) < 2e-2


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_split_tail_ragged_batch(cuda_device, mode):
    H = 16
    shapes = [(4096, 3000), (2048, 100), (1000, 700)]
    reqs = [make_request(T, P, H, seed=950 + i, device=cuda_device, cap=P, mode=mode)
            for i, (T, P) in enumerate(shapes)]
    ws = bca.step_workspace(cuda_device)
    o, cu = run_batch(reqs, H, cuda_device, workspace=ws)
    tol = REL_L2_FP8 if mode != "bf16" else 5e-3
    for i, r in enumerate(reqs):
        rows = sample_rows(r["T"], 64, seed=i)
        got = o[cu[i]:cu[i + 1]][torch.from_numpy(rows).to(cuda_device)]
        assert_parity(got, oracle_for(r, rows=rows), rel_l2=tol, what=f"req {i}")


def test_workspace_too_small_means_no_split(cuda_device):
    H = 32
    req = make_request(4096, 512, H, seed=901, device=cuda_device)
    tiny = torch.empty(1024, dtype=torch.uint8, device=cuda_device)
    o, _ = run_batch([req], H, cuda_device, workspace=tiny)
    rows = sample_rows(4096, 64, seed=3)
    assert_parity(o[torch.from_numpy(rows).to(cuda_device)], oracle_for(req, rows=rows))


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_many_items_per_cta_with_half_empty_q_pairs(cuda_device, mode):
    """T = 128 per request: every unit has an empty second Q tile; H = 256 and two
    requests give 512 items, several per CTA (with and without the split round)."""
    H = 256
    reqs = [make_request(128, 200, H, seed=980 + i, device=cuda_device, mode=mode)
            for i in range(2)]
    tol = REL_L2_FP8 if mode != "bf16" else 5e-3
    for ws in (None, bca.step_workspace(cuda_device)):
        o, cu = run_batch(reqs, H, cuda_device, workspace=ws)
        for i, r in enumerate(reqs):
            rows = sample_rows(128, 24, seed=i)
            got = o[cu[i]:cu[i + 1]][torch.from_numpy(rows).to(cuda_device)]
            assert_parity(got, oracle_for(r, rows=rows), rel_l2=tol, what=f"req {i}")


@pytest.mark.parametrize("n_req,mode", [(9, "bf16"), (64, "bf16"), (64, "fp8")])
def test_batches_beyond_eight_requests(cuda_device, n_req, mode):
    """Batches of 9..64 requests take the largest parameter block (64 requests per
    launch, the call's maximum); ragged T and P, empty requests included, with and
    without the split round."""
    H = 2
    rng = np.random.default_rng(n_req)
    # every seventh request of the 64 is empty (9 requests: none, so that all of
    # them reach the kernel)
    shapes = [(0 if (n_req > 9 and i % 7 == 3) else int(rng.integers(1, 300)),
               int(rng.integers(0, 400))) for i in range(n_req)]
    reqs = [make_request(T, P, H, seed=1200 + i, device=cuda_device, cap=P + 2, mode=mode)
            for i, (T, P) in enumerate(shapes)]
    tol = REL_L2_FP8 if mode != "bf16" else 5e-3
    for ws in (None, bca.step_workspace(cuda_device)):
        o, cu = run_batch(reqs, H, cuda_device, workspace=ws)
        for i, r in enumerate(reqs):
            if r["T"] == 0:
                continue
            assert_parity(o[cu[i]:cu[i + 1]], oracle_for(r), rel_l2=tol, what=f"req {i}")


def test_binding_rejects_tensors_the_kernels_cannot_read(cuda_device):
    """Wrong dtype, a non-contiguous view, mismatched shapes, target rows beyond the
    tensors, a slot on the wrong side of cu_target: BCA_ERR_INVALID_ARG from the
    binding, nothing enqueued, and the library still works afterwards."""
    req = make_request(256, 128, 2, seed=1300, device=cuda_device)
    q, k, v, slot = req["q"], req["k"], req["v"], req["slot"]
    o = torch.empty_like(q)
    bad = [
        (q.float(), k, v, o, [0, 256]),
        (q.transpose(0, 1).contiguous().transpose(0, 1), k, v, o, [0, 256]),
        (q, k[:255], v, o, [0, 256]),
        (q, k, v, o, [0, 300]),
        (q, k, v, o, [0, 100, 256]),
    ]
    for args in bad:
        with pytest.raises(bca.BcaError) as e:
            bca.step_attend(*args, [slot], SCALE)
        assert e.value.status == 1
    with pytest.raises(bca.BcaError):
        bca.kv_store(k.float(), v, 128, slot, epoch=3)
    with pytest.raises(bca.BcaError):
        bca.kv_store(k[:100], v[:100], 128, slot, epoch=3)  # fewer rows than the prefix
    o2, _ = run_batch([req], 2, cuda_device)
    assert_parity(o2, oracle_for(req), what="after rejected calls")
