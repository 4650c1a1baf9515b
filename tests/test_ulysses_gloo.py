"""Head-sharded (Ulysses) protocol on CPU with gloo ranks ("Qwen/Qwen-Image-2.1",
"Overview" / "Limitations": the engine's sequence parallelism is Ulysses).

Every rank holds a block of rows of all heads; after seq_to_head it must hold all
rows of its heads, head_to_seq must invert that, and a cached step computed per head
shard (here by the oracle, which treats every (row, head) independently) and
returned to the row blocks must equal the unsharded result exactly.  The layout
copies are test-side torch permutations (the library's pack/unpack kernels are
checked against the same permutations on the GPU); the exchange is the real
all_to_all_single of the process group."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torch_pack(x, send, n):
    rows, H, d = x.shape
    send.copy_(x.view(rows, n, H // n, d).permute(1, 0, 2, 3))


def torch_unpack(recv, x, n):
    rows, H, d = x.shape
    x.copy_(recv.permute(1, 0, 2, 3).reshape(rows, H, d))


def _full(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _worker(rank, world, port, out):
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        import oracle
        from block_causal_attention_dit_b200.ulysses import ShardPlan, Ulysses
        H, d, P = 4 * world, 128, 24
        cu = [0, 40, 64]  # two requests, packed
        T = cu[-1]
        plan = ShardPlan(world, rank, T, H)
        u = Ulysses(plan, pack=torch_pack, unpack=torch_unpack)
        q, k, v = (_full((T, H, d), 10 + i) for i in range(3))
        caches = [(_full((H, P, d), 20 + 2 * r), _full((H, P, d), 21 + 2 * r)) for r in range(2)]
        r0, r1 = plan.row_range
        h0, h1 = plan.head_range
        res = {}
        qh = u.seq_to_head(q[r0:r1].contiguous())
        res["seq_to_head"] = bool(torch.equal(qh, q[:, h0:h1]))
        back = torch.empty_like(q[r0:r1])
        u.head_to_seq(qh, back)
        res["round_trip"] = bool(torch.equal(back, q[r0:r1]))
        # cached step on this rank's heads (oracle as the attention), back to row blocks
        kh, vh = (u.seq_to_head(x[r0:r1].contiguous()) for x in (k, v))
        scale = 1.0 / math.sqrt(d)
        oh = torch.empty((T, H // world, d), dtype=torch.float64)
        for r in range(2):
            sl = slice(cu[r], cu[r + 1])
            oh[sl] = torch.from_numpy(oracle.cached_step(
                qh[sl], kh[sl], vh[sl], caches[r][0][h0:h1].contiguous(),
                caches[r][1][h0:h1].contiguous(), P, scale))
        o_local = torch.empty((r1 - r0, H, d), dtype=torch.float64)
        u.head_to_seq(oh, o_local)
        want = np.concatenate([oracle.cached_step(q[cu[r]:cu[r + 1]], k[cu[r]:cu[r + 1]],
                                                  v[cu[r]:cu[r + 1]], caches[r][0], caches[r][1],
                                                  P, scale) for r in range(2)])
        res["step_equals_unsharded"] = bool(np.array_equal(o_local.numpy(), want[r0:r1]))
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_protocol_gloo(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert len(res) == world
    for r in range(world):
        assert res[r] == {"seq_to_head": True, "round_trip": True,
                          "step_equals_unsharded": True}, (r, res[r])


def test_shard_plan_checks():
    from block_causal_attention_dit_b200.ulysses import ShardPlan
    p = ShardPlan(4, 3, 4096, 32)
    assert p.row_range == (3072, 4096) and p.head_range == (24, 32)
    with pytest.raises(ValueError):
        ShardPlan(3, 0, 4096, 32)
    with pytest.raises(ValueError):
        ShardPlan(2, 2, 4096, 32)
