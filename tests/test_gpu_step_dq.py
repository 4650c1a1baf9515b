"""bca_step_attend_dq: the cached step over an e4m3 prefix cache ("Qwen/Qwen-Image-
2.1" vLLM recipe, "Prefix KV cache": "fp8_v" and "fp8") with each cache tensor
expanded to bf16 once per call, before the attention.  The expansion is exact and
the attention folds the per-head scales in as bca_step_attend does, so the output
equals bca_step_attend's on the same slots bit for bit; it is also checked against
the oracle reading the same bytes (rel-L2 <= 2e-2, the e4m3-cache rule)."""
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


def _batch(shapes, H, mode, device, seed):
    reqs = []
    for i, (T, P) in enumerate(shapes):
        q, k, v = (randn_bf16((T, H, 128), seed + 10 * i + t, device) for t in range(3))
        # K scaled per request (different per-head scales and sharper softmax rows)
        pk = randn_bf16((max(P, 1), H, 128), seed + 10 * i + 5, device) * (1 + i)
        pv = randn_bf16((max(P, 1), H, 128), seed + 10 * i + 6, device)
        slot = bca.KVSlot(P + 7, H, mode)
        slot.buffer.fill_(0xFF)  # NaN codes past the prefix: never read
        bca.kv_store(pk, pv, P, slot, epoch=1)
        reqs.append(dict(q=q, k=k, v=v, slot=slot, T=T, P=P))
    cu = np.concatenate([[0], np.cumsum([r["T"] for r in reqs])]).tolist()
    cat = lambda n: torch.cat([r[n] for r in reqs])
    return reqs, cu, cat("q"), cat("k"), cat("v")


@pytest.mark.parametrize("mode", ["fp8", "fp8_v"])
@pytest.mark.parametrize("split", [False, True])
def test_equals_step_attend_bitwise_and_oracle(cuda_device, mode, split):
    H = 4
    shapes = [(300, 513), (77, 0), (0, 20), (256, 1), (130, 2000), (1024, 2500)]
    reqs, cu, q, k, v = _batch(shapes, H, mode, cuda_device, 7000)
    slots = [r["slot"] for r in reqs]
    ws = bca.step_workspace(cuda_device) if split else None
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ref, out = torch.empty_like(q), torch.full_like(q, float("nan"))
    bca.step_attend(q, k, v, ref, cu, slots, SCALE, workspace=ws, dev_status=status)
    scratch = bca.step_attend_dq(q, k, v, out, cu, slots, SCALE, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert scratch.numel() >= bca.step_dq_scratch_bytes(slots)
    assert torch.equal(out, ref)
    for i, r in enumerate(reqs):
        if r["T"] == 0:
            continue
        s = r["slot"]
        kk = oracle.KIND_E4M3 if mode == "fp8" else oracle.KIND_BF16
        want = oracle.cached_step(r["q"], r["k"], r["v"], s.k_view().cpu(), s.v_view().cpu(),
                                  r["P"], SCALE, k_kind=kk, v_kind=oracle.KIND_E4M3,
                                  k_scale=s.k_scale_view().cpu().numpy(),
                                  v_scale=s.v_scale_view().cpu().numpy())
        assert_parity(out[cu[i]:cu[i + 1]], want, rel_l2=REL_L2_FP8, what=f"dq {mode} req {i}")


def test_expanded_scratch_holds_the_decoded_codes(cuda_device):
    """The scratch holds, per request, [H, n_tokens, 128] bf16 of K then V: the exact
    OFP8 E4M3 values of the codes (the oracle's decoder), scales not applied."""
    H = 3
    reqs, cu, q, k, v = _batch([(128, 300), (64, 129)], H, "fp8", cuda_device, 7100)
    slots = [r["slot"] for r in reqs]
    out = torch.empty_like(q)
    scratch = bca.step_attend_dq(q, k, v, out, cu, slots, SCALE)
    torch.cuda.synchronize()
    table = np.array([oracle.e4m3_decode(c) for c in range(256)])
    off = 0
    for r in reqs:
        P = r["P"]
        nbytes = H * P * 128 * 2
        for codes in (r["slot"].k_view(), r["slot"].v_view()):
            got = scratch[off:off + nbytes].view(torch.bfloat16).view(H, P, 128)
            want = table[codes[:, :P].cpu().numpy()]
            assert np.array_equal(got.double().cpu().numpy(), want)
            off += (nbytes + 255) // 256 * 256


def test_serving_batch_sampled_rows(cuda_device):
    """The 8-request serving workload (e4m3 K and V) in the benchmark's configuration:
    bit-identical to bca_step_attend; sampled rows of every request against the
    oracle."""
    wl = W.workload(4)
    dev = cuda_device
    slots, qs, ks_, vs_ = [], [], [], []
    for i, r in enumerate(wl.requests):
        q0, k0, v0 = W.qkv(wl, 0, 0, i, dev)
        slot = bca.KVSlot(r.prefix, wl.heads, "fp8")
        bca.kv_store(k0, v0, r.prefix, slot, epoch=1)
        slots.append(slot)
        del q0, k0, v0
        q, k, v = W.qkv(wl, 0, 1, i, dev)
        qs.append(q), ks_.append(k), vs_.append(v)
    q, k, v = torch.cat(qs), torch.cat(ks_), torch.cat(vs_)
    cu = np.concatenate([[0], np.cumsum([r.target for r in wl.requests])]).tolist()
    ws = bca.step_workspace(dev)
    ref, out = torch.empty_like(q), torch.empty_like(q)
    bca.step_attend(q, k, v, ref, cu, slots, wl.scale, workspace=ws)
    bca.step_attend_dq(q, k, v, out, cu, slots, wl.scale, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    for i, r in enumerate(wl.requests):
        rows = sample_rows(r.target, 8, seed=i, boundaries=(128, 2048))
        s = slots[i]
        want = oracle.cached_step(qs[i], ks_[i], vs_[i], s.k_view().cpu(), s.v_view().cpu(),
                                  r.prefix, wl.scale, k_kind=oracle.KIND_E4M3,
                                  v_kind=oracle.KIND_E4M3, k_scale=s.k_scale_view().cpu().numpy(),
                                  v_scale=s.v_scale_view().cpu().numpy(), rows=rows)
        got = out[cu[i]:cu[i + 1]][torch.from_numpy(rows).to(dev)]
        assert_parity(got, want, rel_l2=REL_L2_FP8, what=f"serving dq request {i}")


def test_argument_errors(cuda_device):
    H = 2
    reqs, cu, q, k, v = _batch([(64, 32)], H, "fp8", cuda_device, 7200)
    o = torch.empty_like(q)
    bf = bca.KVSlot(32, H, "bf16")
    bca.kv_store(k[:32], v[:32], 32, bf, epoch=1)
    with pytest.raises(bca.BcaError) as e:
        bca.step_attend_dq(q, k, v, o, cu, [bf], SCALE)
    assert e.value.status == 2
    small = torch.empty(256, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(bca.BcaError) as e:
        bca.step_attend_dq(q, k, v, o, cu, [reqs[0]["slot"]], SCALE, dq_scratch=small)
    assert e.value.status == 3
