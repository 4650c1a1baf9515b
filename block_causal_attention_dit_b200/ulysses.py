"""Head-sharded (Ulysses) sequence parallelism around the attention calls.

"Qwen/Qwen-Image-2.1" (recipes.vllm.ai), "Overview" and "Limitations": the
engine's sequence parallelism is Ulysses.  N ranks each hold a contiguous block of
rows_local = rows / N rows (all H heads) of Q, K, V.  One all-to-all per tensor
gives every rank all rows of its H/N heads; bca_prefill / bca_step_attend run on
that head shard (a rank's cache slots hold its H/N heads, so cached steps move no
prefix K/V at all); one all-to-all returns O to the row blocks.

The copies around the exchange run in the library (bca_ulysses_pack / unpack); the
exchange itself is torch.distributed.all_to_all_single on the caller's process
group (NCCL over NVLink on GPUs).  This module only sizes buffers and orders the
calls.  `exchange` and `pack`/`unpack` can be replaced (tests do this to run the
same protocol with gloo on CPU tensors).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

import block_causal_attention_dit_b200 as bca


@dataclass
class ShardPlan:
    """Row and head ranges of one rank."""
    n_ranks: int
    rank: int
    rows: int        # all rows (packed over requests)
    heads: int

    def __post_init__(self):
        if self.n_ranks < 1 or not 0 <= self.rank < self.n_ranks:
            raise ValueError("bad rank / world size")
        if self.rows % self.n_ranks or self.heads % self.n_ranks:
            raise ValueError(f"rows ({self.rows}) and heads ({self.heads}) must be multiples "
                             f"of the number of ranks ({self.n_ranks})")

    @property
    def rows_local(self) -> int:
        return self.rows // self.n_ranks

    @property
    def heads_local(self) -> int:
        return self.heads // self.n_ranks

    @property
    def row_range(self):
        return self.rank * self.rows_local, (self.rank + 1) * self.rows_local

    @property
    def head_range(self):
        return self.rank * self.heads_local, (self.rank + 1) * self.heads_local


def _dist_exchange(group):
    import torch.distributed as dist

    def exchange(recv, send):
        dist.all_to_all_single(recv, send, group=group)
    return exchange


class Ulysses:
    """seq_to_head / head_to_seq and the attention calls on a head shard."""

    def __init__(self, plan: ShardPlan, group=None,
                 exchange: Optional[Callable] = None,
                 pack: Optional[Callable] = None, unpack: Optional[Callable] = None):
        self.plan = plan
        self.exchange = exchange or _dist_exchange(group)
        self.pack = pack or bca.ulysses_pack
        self.unpack = unpack or bca.ulysses_unpack

    def seq_to_head(self, x_local):
        """[rows_local, H, d] (this rank's rows) -> [rows, H/N, d] (this rank's heads)."""
        import torch
        p = self.plan
        send = torch.empty((p.n_ranks, p.rows_local, p.heads_local, x_local.shape[2]),
                           dtype=x_local.dtype, device=x_local.device)
        self.pack(x_local, send, p.n_ranks)
        recv = torch.empty_like(send)
        self.exchange(recv, send)
        return recv.view(p.rows, p.heads_local, x_local.shape[2])

    def head_to_seq(self, y_head, out_local):
        """[rows, H/N, d] (this rank's heads) -> out_local [rows_local, H, d]."""
        import torch
        p = self.plan
        send = y_head.reshape(p.n_ranks, p.rows_local, p.heads_local, y_head.shape[2])
        recv = torch.empty_like(send)
        self.exchange(recv, send)
        self.unpack(recv, out_local, p.n_ranks)
        return out_local

    def prefill(self, q_l, k_l, v_l, o_l, block_offsets, scale, slot=None, epoch=0,
                dev_status=None):
        """Block-causal prefill of one request whose rows are sharded over the ranks
        (slot: this rank's H/N-head cache slot)."""
        import torch
        q, k, v = (self.seq_to_head(x) for x in (q_l, k_l, v_l))
        o = torch.empty_like(q)
        bca.prefill(q, k, v, o, block_offsets, scale, slot=slot, epoch=epoch,
                    dev_status=dev_status)
        return self.head_to_seq(o, o_l)

    def step_attend(self, q_l, k_l, v_l, o_l, cu_target, slots, scale, workspace=None,
                    dev_status=None):
        """Cached step of a packed same-phase batch whose packed target rows are
        sharded over the ranks (slots: this rank's H/N-head slots, one per request)."""
        import torch
        q, k, v = (self.seq_to_head(x) for x in (q_l, k_l, v_l))
        o = torch.empty_like(q)
        bca.step_attend(q, k, v, o, cu_target, slots, scale, workspace=workspace,
                        dev_status=dev_status)
        return self.head_to_seq(o, o_l)
