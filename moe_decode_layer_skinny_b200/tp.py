"""Tensor-parallel decode layer over a torch.distributed process group.

The layer is sharded over the R ranks of a group as the pages shard it over
the GPUs of a node (wireai.ir "vLLM Blackwell Kimi decode", section "4 key
changes", item 2: the o-proj partial sums are reduced across GPUs together
with the residual; item 3: the router scores are split among the
tensor-parallel ranks; bigchange.ai "where the time went": the shared expert
beside the routed ones).  Rank r of R owns

  * q heads [r Hq/R, (r+1) Hq/R) and the kv heads they read: its rows of the
    QKV projection and its columns of the o-proj input;
  * experts [r E/R, (r+1) E/R) of the router;
  * intermediate rows [r I/R, (r+1) I/R) of every expert (shared and routed):
    gate/up rows and down columns.

One decode step is four local phases and three exchanges:

  1. p_r = Wo[:, cols_r] a[:, cols_r]  (and the rank's QKV rows)
     all-reduce(sum) p                              -> h1 = x + sum_r p_r
  2. logits[:, E_r] = Wr[E_r] h1 (+ b)
     all-gather logits                              -> the same selection on
                                                       every rank
  3. y_r = shared_r(h1) + s sum_j g_j expert_{j,r}(h1)
     all-reduce(sum) y
  4. hidden = h1 + sum_r y_r

The phases are the shard object's methods (``ShardOps``); this module only
orders them and moves the partial sums between ranks with the group's
collectives (NCCL over NVLink on GPUs, gloo on CPU).  Every rank takes the
same collective steps in the same order.
"""
from __future__ import annotations

from typing import Protocol


class ShardOps(Protocol):
    """One rank's share of the layer (see the module docstring)."""

    def attn_partial(self, hidden, attn):
        """Phase 1: this rank's o-proj partial sum p_r [M, H] (fp32 or wider);
        also computes the rank's QKV rows."""

    def router_shard(self, hidden, p_sum):
        """Phase 2: h1 = x + p_sum (kept by the shard); logits of the rank's
        experts [M, E/R]."""

    def moe_partial(self, logits):
        """Phase 3: selection from the gathered logits [M, E]; the rank's
        expert partial sum y_r [M, H]."""

    def combine(self, y_sum, hidden):
        """Phase 4: hidden = h1 + y_sum, in place."""


def decode_tp(shard: ShardOps, hidden, attn, group=None):
    """One decode step of the sharded layer on this rank.  ``hidden`` [M, H]
    is replicated on every rank and updated in place; ``attn`` [M, A] is the
    attention output, replicated (each rank reads its own columns)."""
    import torch
    import torch.distributed as dist

    R = dist.get_world_size(group)
    p = shard.attn_partial(hidden, attn)
    dist.all_reduce(p, op=dist.ReduceOp.SUM, group=group)
    ls = shard.router_shard(hidden, p)
    parts = [torch.empty_like(ls) for _ in range(R)]
    dist.all_gather(parts, ls.contiguous(), group=group)
    logits = torch.cat(parts, dim=1)
    y = shard.moe_partial(logits)
    dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    shard.combine(y, hidden)
    return hidden


class _DeviceArray:
    """A layer-owned device buffer as a CUDA array interface (fp32, 2-D)."""

    def __init__(self, ptr: int, shape):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": "<f4",
                                         "data": (int(ptr), False), "version": 3, "strides": None}


class CudaShard:
    """ShardOps on one tensor-parallel shard of the CUDA layer (a
    ``moe_decode_layer_skinny_b200.Layer`` created with tp_rank / tp_size):
    the phases are its kd_tp_* calls; the partial sums live in the layer's
    exchange buffers, which the collectives reduce in place."""

    def __init__(self, layer, M: int):
        import torch
        self.layer, self.M = layer, M
        s = layer.spec
        R = s.tp_size
        b = layer.tp_buffers()
        dev = torch.device("cuda", torch.cuda.current_device())
        self.p = torch.as_tensor(_DeviceArray(b["p"], (M, s.hidden)), device=dev)
        self.lshard = torch.as_tensor(_DeviceArray(b["lshard"], (M, s.n_experts // R)), device=dev)
        self.lfull = torch.as_tensor(_DeviceArray(b["lfull"], (M, s.n_experts)), device=dev)
        self.y = torch.as_tensor(_DeviceArray(b["y"], (M, s.hidden)), device=dev)

    def attn_partial(self, hidden, attn):
        self.layer.tp_attn(hidden, attn, self.M)
        return self.p

    def router_shard(self, hidden, p_sum):
        if p_sum.data_ptr() != self.p.data_ptr():
            self.p.copy_(p_sum)
        self.layer.tp_router(hidden, self.M)
        return self.lshard

    def moe_partial(self, logits):
        self.lfull.copy_(logits)
        self.layer.tp_moe(self.M)
        return self.y

    def combine(self, y_sum, hidden):
        if y_sum.data_ptr() != self.y.data_ptr():
            self.y.copy_(y_sum)
        self.layer.tp_combine(hidden, self.M)
