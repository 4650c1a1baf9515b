"""bca_kv_store on the GPU against the oracle: bf16 copies exact, e4m3 cache bytes
and per-head scales bit-exact ("Qwen/Qwen-Image-2.1" vLLM recipe, "Prefix KV
cache": "fp8_v" quantises V only, "fp8" K and V)."""
import numpy as np
import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200.workloads import randn_bf16

pytestmark = pytest.mark.gpu


def _fill_sentinel(slot):
    slot.buffer.fill_(0x5A)


@pytest.mark.parametrize("P,H,cap", [(128, 4, 128), (77, 3, 200), (1, 2, 5), (513, 32, 600)])
def test_bf16_copy_exact(cuda_device, P, H, cap):
    k = randn_bf16((P + 9, H, 128), 11, cuda_device)
    v = randn_bf16((P + 9, H, 128), 12, cuda_device)
    slot = bca.KVSlot(cap, H, "bf16")
    _fill_sentinel(slot)
    bca.kv_store(k, v, P, slot, epoch=7)
    torch.cuda.synchronize()
    assert slot.n_tokens == P and slot.epoch == 7
    assert torch.equal(slot.k_view()[:, :P], k[:P].permute(1, 0, 2))
    assert torch.equal(slot.v_view()[:, :P], v[:P].permute(1, 0, 2))
    # rows beyond the prefix are untouched
    tail = slot.k_view()[:, P:].contiguous().view(torch.uint8)
    assert bool((tail == 0x5A).all())


@pytest.mark.parametrize("mode", ["fp8", "fp8_v"])
@pytest.mark.parametrize("P,H,cap,amp", [(128, 4, 128, 1.0), (77, 3, 100, 37.0),
                                         (1000, 32, 1024, 0.01), (3, 2, 3, 300.0)])
def test_fp8_bytes_and_scales_bit_exact(cuda_device, mode, P, H, cap, amp):
    k = (randn_bf16((P, H, 128), 21, cuda_device).float() * amp).to(torch.bfloat16)
    v = (randn_bf16((P, H, 128), 22, cuda_device).float() * amp * 0.5).to(torch.bfloat16)
    slot = bca.KVSlot(cap, H, mode)
    _fill_sentinel(slot)
    bca.kv_store(k, v, P, slot, epoch=3)
    torch.cuda.synchronize()
    vc, vs = oracle.quantize_prefix(v.cpu(), P, cap)
    assert np.array_equal(slot.v_view()[:, :P].cpu().numpy(), vc[:, :P])
    assert np.array_equal(slot.v_scale_view().cpu().numpy(), vs)
    if mode == "fp8":
        kc, ks = oracle.quantize_prefix(k.cpu(), P, cap)
        assert np.array_equal(slot.k_view()[:, :P].cpu().numpy(), kc[:, :P])
        assert np.array_equal(slot.k_scale_view().cpu().numpy(), ks)
    else:
        assert torch.equal(slot.k_view()[:, :P], k.permute(1, 0, 2))


def test_fp8_strided_source_and_zero_head(cuda_device):
    P, H = 300, 4
    big = randn_bf16((P, H * 128 + 64), 31, cuda_device)
    big[:, 128:256] = 0  # head 1 all zeros -> scale 1, codes 0
    k = big[:, : H * 128]
    v = big[:, 64: 64 + H * 128]
    slot = bca.KVSlot(P, H, "fp8")
    bca.kv_store(k, v, P, slot, epoch=1, row_stride=big.stride(0))
    torch.cuda.synchronize()
    kc, ks = oracle.quantize_prefix(k.contiguous().view(P, H, 128).cpu(), P)
    vc, vs = oracle.quantize_prefix(v.contiguous().view(P, H, 128).cpu(), P)
    assert ks[1] == 1.0 and (kc[1] == 0).all()
    assert np.array_equal(slot.k_view().cpu().numpy(), kc)
    assert np.array_equal(slot.v_view().cpu().numpy(), vc)
    assert np.array_equal(slot.k_scale_view().cpu().numpy(), ks)
    assert np.array_equal(slot.v_scale_view().cpu().numpy(), vs)


def test_restore_for_a_new_request(cuda_device):
    """Per-request rebuild: a slot reused by a shorter second request holds exactly
    the second request's prefix (its epoch and length), never the first's."""
    H = 2
    slot = bca.KVSlot(256, H, "fp8")
    a = randn_bf16((200, H, 128), 41, cuda_device)
    b = randn_bf16((60, H, 128), 42, cuda_device) * 3
    bca.kv_store(a, a, 200, slot, epoch=1)
    bca.kv_store(b, b, 60, slot, epoch=2)
    torch.cuda.synchronize()
    assert slot.epoch == 2 and slot.n_tokens == 60
    bc, bs = oracle.quantize_prefix(b.cpu(), 60)
    assert np.array_equal(slot.k_view()[:, :60].cpu().numpy(), bc)
    assert np.array_equal(slot.k_scale_view().cpu().numpy(), bs)


def test_empty_prefix_only_stamps(cuda_device):
    slot = bca.KVSlot(16, 2, "bf16")
    x = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device=cuda_device)
    bca.kv_store(x, x, 0, slot, epoch=5)
    assert slot.n_tokens == 0 and slot.epoch == 5


def test_fp8_heads_with_tiny_and_huge_amax_bit_exact(cuda_device):
    """Heads whose absmax is below 2^-95 take the encoder's correctly rounded
    division (the reciprocal would leave the normal range); a head near the top of
    the bf16 range takes the fast one.  Bytes and scales equal the oracle's."""
    P, H = 200, 4
    base = randn_bf16((P, H, 128), 41, cuda_device).float()
    base[::7, :, ::5] = -0.0  # negative zeros keep their sign in the codes (0x80)
    factors = torch.tensor([2.0 ** -120, 2.0 ** -100, 1.0, 2.0 ** 100], device=cuda_device)
    k = (base * factors[None, :, None]).to(torch.bfloat16)
    v = (base.flip(0) * factors.flip(0)[None, :, None]).to(torch.bfloat16)
    slot = bca.KVSlot(P, H, "fp8")
    bca.kv_store(k, v, P, slot, epoch=1)
    torch.cuda.synchronize()
    for x, codes, scales in ((k, slot.k_view(), slot.k_scale_view()),
                             (v, slot.v_view(), slot.v_scale_view())):
        want_c, want_s = oracle.quantize_prefix(x.cpu(), P, P)
        assert np.array_equal(codes.cpu().numpy(), want_c)
        assert np.array_equal(scales.cpu().numpy(), want_s)


def test_encoder_division_matches_correct_rounding_exhaustively(cuda_device):
    """The e4m3 encoder divides by the head's scale with a reciprocal and one
    FMA-residual correction (Markstein's scheme), or, for heads with amax below
    2^-95, with the correctly rounded division.  For every positive finite bf16 amax
    and every bf16 x with |x| <= amax (about 10^9 pairs), the resulting e4m3 code
    equals the code of the correctly rounded fp32 quotient."""
    assert bca.selftest_e4m3_division(cuda_device) == 0


def test_batch_store_equals_oracle_per_request(cuda_device):
    """bca_kv_store_batch: the requests of a batch (different prefix lengths, head
    counts and cache dtypes) in one launch; every slot's bytes and scales equal the
    oracle's, rows past the prefix untouched, every slot stamped."""
    specs = [(1500, 32, "fp8", 1600), (77, 32, "fp8", 80), (640, 8, "bf16", 700),
             (300, 4, "fp8_v", 300), (0, 4, "fp8", 16), (5000, 2, "fp8", 5000)]
    items, srcs = [], []
    for i, (P, H, mode, cap) in enumerate(specs):
        k = randn_bf16((max(P, 1), H, 128), 500 + 2 * i, cuda_device) * (1 + i)
        v = randn_bf16((max(P, 1), H, 128), 501 + 2 * i, cuda_device) * 0.3
        slot = bca.KVSlot(cap, H, mode)
        _fill_sentinel(slot)
        items.append((k, v, P, slot))
        srcs.append((k, v))
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bca.kv_store_batch(items, epoch=9, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (k, v, P, slot), (P_, H, mode, cap) in zip(items, specs):
        assert slot.n_tokens == P and slot.epoch == 9
        for x, codes, scales, q in ((k, slot.k_view(), slot.k_scale_view(), mode == "fp8"),
                                    (v, slot.v_view(), slot.v_scale_view(), mode != "bf16")):
            if P == 0:
                continue
            if q:
                want_c, want_s = oracle.quantize_prefix(x.cpu(), P, cap)
                assert np.array_equal(codes[:, :P].cpu().numpy(), want_c[:, :P]), (P, mode)
                assert np.array_equal(scales.cpu().numpy(), want_s), (P, mode)
            else:
                assert torch.equal(codes[:, :P], x[:P].permute(1, 0, 2)), (P, mode)
            tail = codes[:, P:].contiguous().view(torch.uint8)
            assert bool((tail == 0x5A).all()), (P, mode)


def test_batch_store_rejects_a_repeated_slot(cuda_device):
    k = randn_bf16((64, 2, 128), 600, cuda_device)
    slot = bca.KVSlot(64, 2, "fp8")
    with pytest.raises(bca.BcaError) as e:
        bca.kv_store_batch([(k, k, 64, slot), (k, k, 32, slot)], epoch=1)
    assert e.value.status == 1
    assert slot.epoch == 0


def test_non_finite_input_reports_status(cuda_device):
    """Inputs must be finite.  An e4m3 tensor with an Inf in one head reports
    BCA_ERR_NONFINITE through dev_status; the other heads are still encoded
    exactly.  A bf16 copy of the same rows is exact and reports nothing."""
    P, H = 257, 4
    k = randn_bf16((P, H, 128), 610, cuda_device)
    v = randn_bf16((P, H, 128), 611, cuda_device)
    k[100, 2, 7] = float("inf")
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    slot = bca.KVSlot(P, H, "fp8")
    bca.kv_store(k, v, P, slot, epoch=1, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 7  # BCA_ERR_NONFINITE
    kc, ks = oracle.quantize_prefix(k.cpu(), P)
    for h in (0, 1, 3):
        assert np.array_equal(slot.k_view()[h].cpu().numpy(), kc[h])
        assert slot.k_scale_view()[h].item() == ks[h]
    vc, vs = oracle.quantize_prefix(v.cpu(), P)
    assert np.array_equal(slot.v_view().cpu().numpy(), vc)
    status.zero_()
    s16 = bca.KVSlot(P, H, "bf16")
    bca.kv_store(k, v, P, s16, epoch=1, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(s16.k_view(), k.permute(1, 0, 2))


def test_batch_store_many_columns_per_cluster(cuda_device):
    """512 e4m3 columns in one launch (8 requests x K and V x 32 heads): every
    cluster of the store kernel takes a dozen or more columns in turn, so the
    interleaving of one column's encode pass with the next column's absmax pass and
    the rotation of the rank-exchange buffers over many columns both run.  Bytes and
    scales equal the oracle's for every slot."""
    prefixes = [611, 97, 420, 333, 800, 5, 256, 129]
    items = []
    for i, P in enumerate(prefixes):
        k = randn_bf16((P, 32, 128), 700 + 2 * i, cuda_device) * (0.5 + i)
        v = randn_bf16((P, 32, 128), 701 + 2 * i, cuda_device) * (3.0 / (1 + i))
        slot = bca.KVSlot(P + 3, 32, "fp8")
        _fill_sentinel(slot)
        items.append((k, v, P, slot))
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bca.kv_store_batch(items, epoch=4, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for k, v, P, slot in items:
        for x, codes, scales in ((k, slot.k_view(), slot.k_scale_view()),
                                 (v, slot.v_view(), slot.v_scale_view())):
            want_c, want_s = oracle.quantize_prefix(x.cpu(), P, P + 3)
            assert np.array_equal(codes[:, :P].cpu().numpy(), want_c[:, :P]), P
            assert np.array_equal(scales.cpu().numpy(), want_s), P
            assert bool((codes[:, P:].contiguous().view(torch.uint8) == 0x5A).all()), P


def test_batch_store_bf16_row_pieces(cuda_device):
    """Few long bf16 heads are cut into row pieces across clusters (here 4 heads of
    5000 rows, and the bf16 K of an "fp8_v" slot next to its e4m3 V): the copies are
    exact, the e4m3 V bit-exact, and nothing past the prefix is written."""
    specs = [(5000, 4, "bf16", 5004), (3001, 4, "fp8_v", 3001)]
    items = []
    for i, (P, H, mode, cap) in enumerate(specs):
        k = randn_bf16((P, H, 128), 720 + 2 * i, cuda_device)
        v = randn_bf16((P, H, 128), 721 + 2 * i, cuda_device) * 7.0
        slot = bca.KVSlot(cap, H, mode)
        _fill_sentinel(slot)
        items.append((k, v, P, slot, mode, cap))
    bca.kv_store_batch([it[:4] for it in items], epoch=2)
    torch.cuda.synchronize()
    for k, v, P, slot, mode, cap in items:
        assert torch.equal(slot.k_view()[:, :P], k.permute(1, 0, 2)), mode
        if mode == "bf16":
            assert torch.equal(slot.v_view()[:, :P], v.permute(1, 0, 2))
        else:
            want_c, want_s = oracle.quantize_prefix(v.cpu(), P, cap)
            assert np.array_equal(slot.v_view()[:, :P].cpu().numpy(), want_c[:, :P])
            assert np.array_equal(slot.v_scale_view().cpu().numpy(), want_s)
        for codes in (slot.k_view(), slot.v_view()):
            assert bool((codes[:, P:].contiguous().view(torch.uint8) == 0x5A).all()), mode


def test_serving_store_full_size_sampled_heads(cuda_device):
    """The 8-request serving store at its full size (e4m3 K and V, prefixes 996 ..
    17075 rows, 32 heads: 512 columns in one launch, the call the bench times):
    sixteen sampled (request, tensor, head) columns are bit-exact against the oracle
    quantising that head's rows (codes and scale), and rows past each prefix are
    untouched."""
    from block_causal_attention_dit_b200 import workloads as W
    wl = W.workload(4)
    items, srcs = [], []
    for i, r in enumerate(wl.requests):
        _, k, v = W.qkv(wl, 0, 0, i, cuda_device)
        slot = bca.KVSlot(r.prefix + 5, wl.heads, "fp8")
        _fill_sentinel(slot)
        items.append((k, v, r.prefix, slot))
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bca.kv_store_batch(items, epoch=5, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(44)
    for _ in range(16):
        i = int(rng.integers(len(items)))
        kv = int(rng.integers(2))
        h = int(rng.integers(wl.heads))
        k, v, P, slot = items[i]
        x = (k, v)[kv][:P, h:h + 1, :].cpu()
        want_c, want_s = oracle.quantize_prefix(x, P, P + 5)
        codes = (slot.k_view(), slot.v_view())[kv][h:h + 1]
        scales = (slot.k_scale_view(), slot.v_scale_view())[kv][h:h + 1]
        assert np.array_equal(codes[:, :P].cpu().numpy(), want_c[:, :P]), (i, kv, h)
        assert np.array_equal(scales.cpu().numpy(), want_s), (i, kv, h)
        assert bool((codes[:, P:].contiguous().view(torch.uint8) == 0x5A).all()), (i, kv, h)


def test_edit_store_full_size_bf16(cuda_device):
    """The 4-ref edit's bf16 prefix store at full size (16864 rows x 32 heads, K and
    V: 64 long heads cut into row pieces across the clusters) is an exact copy, and
    nothing past the prefix is written."""
    from block_causal_attention_dit_b200 import workloads as W
    wl = W.workload(2)
    r = wl.requests[0]
    _, k, v = W.qkv(wl, 0, 0, 0, cuda_device)
    slot = bca.KVSlot(r.prefix + 7, wl.heads, "bf16")
    _fill_sentinel(slot)
    bca.kv_store_batch([(k, v, r.prefix, slot)], epoch=3)
    torch.cuda.synchronize()
    P = r.prefix
    assert torch.equal(slot.k_view()[:, :P], k[:P].permute(1, 0, 2))
    assert torch.equal(slot.v_view()[:, :P], v[:P].permute(1, 0, 2))
    for codes in (slot.k_view(), slot.v_view()):
        assert bool((codes[:, P:].contiguous().view(torch.uint8) == 0x5A).all())
