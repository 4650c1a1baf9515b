"""Head-sharded (Ulysses) path on the GPU ("Qwen/Qwen-Image-2.1", "Overview" /
"Limitations": Ulysses sequence parallelism).

 - bca_ulysses_pack / unpack equal the block permutation they are defined as,
   for 1, 2, 4 and 8 ranks (bit-exact byte moves).
 - N ranks emulated on one GPU with the library's pack/unpack and the attention
   kernel on each head shard (the all-to-all done by slicing): the cached step
   returned to the row blocks matches the oracle's unsharded cached step within the
   bf16 tolerance, and is bit-identical to the unsharded call (each (row, head) unit
   computes the same arithmetic whatever the sharding; no split workspace, so no
   schedule-dependent merge).
 - One real rank with NCCL: Ulysses.step_attend through all_to_all_single matches
   the oracle and equals the plain call bit for bit."""
import math
import os
import socket

import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200.ulysses import ShardPlan, Ulysses
from block_causal_attention_dit_b200.workloads import randn_bf16
from _parity import assert_parity

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_pack_unpack_are_the_block_permutation(cuda_device, n):
    rows, H = 333, 32
    x = randn_bf16((rows, H, 128), 40 + n, cuda_device)
    send = torch.empty((n, rows, H // n, 128), dtype=torch.bfloat16, device=cuda_device)
    bca.ulysses_pack(x, send, n)
    want = x.view(rows, n, H // n, 128).permute(1, 0, 2, 3)
    back = torch.empty_like(x)
    bca.ulysses_unpack(send, back, n)
    torch.cuda.synchronize()
    assert torch.equal(send, want)
    assert torch.equal(back, x)
    with pytest.raises(bca.BcaError):
        bca.ulysses_pack(x, send, 3)  # 32 heads do not split over 3 ranks


def _oracle(q, k, v, pk, pv):
    """The oracle's (unsharded) cached step of one request, its cache built on the
    host from the prefix rows."""
    return oracle.cached_step(q.cpu(), k.cpu(), v.cpu(), pk.cpu().permute(1, 0, 2).contiguous(),
                              pv.cpu().permute(1, 0, 2).contiguous(), pk.shape[0], SCALE)


def _slots(prefix_k, prefix_v, heads, device):
    s = bca.KVSlot(prefix_k.shape[0], heads, device=device)
    bca.kv_store(prefix_k, prefix_v, prefix_k.shape[0], s, epoch=1)
    return s


@pytest.mark.parametrize("n", [2, 4])
def test_emulated_ranks_match_oracle_and_unsharded(cuda_device, n):
    H, P = 16, 300
    cu = [0, 512, 1024]
    T = cu[-1]
    q, k, v = (randn_bf16((T, H, 128), 60 + i, cuda_device) for i in range(3))
    pre = [tuple(randn_bf16((P, H, 128), 70 + 2 * r + i, cuda_device) for i in range(2))
           for r in range(2)]
    full_slots = [_slots(pk, pv, H, cuda_device) for pk, pv in pre]
    o_ref = torch.empty_like(q)
    bca.step_attend(q, k, v, o_ref, cu, full_slots, SCALE)
    plans = [ShardPlan(n, r, T, H) for r in range(n)]
    Tl, Hn = T // n, H // n
    # each rank packs its row block of q, k, v
    sends = []
    for p in plans:
        r0, r1 = p.row_range
        per = []
        for x in (q, k, v):
            sb = torch.empty((n, Tl, Hn, 128), dtype=torch.bfloat16, device=cuda_device)
            bca.ulysses_pack(x[r0:r1].contiguous(), sb, n)
            per.append(sb)
        sends.append(per)
    # all-to-all by slicing: rank g receives block g of every rank's send buffer
    o_blocks = []
    for g, p in enumerate(plans):
        qh, kh, vh = (torch.stack([sends[src][i][g] for src in range(n)]).view(T, Hn, 128)
                      for i in range(3))
        h0, h1 = p.head_range
        slots = [_slots(pk[:, h0:h1].contiguous(), pv[:, h0:h1].contiguous(), Hn, cuda_device)
                 for pk, pv in pre]
        oh = torch.empty_like(qh)
        bca.step_attend(qh, kh, vh, oh, cu, slots, SCALE)
        o_blocks.append(oh.view(n, Tl, Hn, 128))
    out = torch.empty_like(q)
    for r, p in enumerate(plans):
        recv = torch.stack([o_blocks[g][r] for g in range(n)])
        r0, r1 = p.row_range
        part = torch.empty((Tl, H, 128), dtype=torch.bfloat16, device=cuda_device)
        bca.ulysses_unpack(recv, part, n)
        out[r0:r1] = part
    torch.cuda.synchronize()
    for r, (pk, pv) in enumerate(pre):
        sl = slice(cu[r], cu[r + 1])
        assert_parity(out[sl], _oracle(q[sl], k[sl], v[sl], pk, pv),
                      what=f"{n} ranks, request {r}")
    assert torch.equal(out, o_ref)


def test_single_rank_nccl_exchange(cuda_device):
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{port}",
                            device_id=cuda_device)
    try:
        H, P, T = 8, 200, 640
        q, k, v = (randn_bf16((T, H, 128), 80 + i, cuda_device) for i in range(3))
        pk, pv = (randn_bf16((P, H, 128), 85 + i, cuda_device) for i in range(2))
        slot = _slots(pk, pv, H, cuda_device)
        o_ref, o = torch.empty_like(q), torch.empty_like(q)
        bca.step_attend(q, k, v, o_ref, [0, T], [slot], SCALE)
        u = Ulysses(ShardPlan(1, 0, T, H))
        u.step_attend(q, k, v, o, [0, T], [slot], SCALE)
        torch.cuda.synchronize()
        assert_parity(o, _oracle(q, k, v, pk, pv), what="one NCCL rank")
        assert torch.equal(o, o_ref)
    finally:
        dist.destroy_process_group()
