"""A ShardOps implementation on the oracle's tensor-parallel slices (fp64 on
CPU), for the tests of the sharded layer's orchestration."""
import numpy as np
import torch

import oracle.tp as otp


class OracleShard:
    def __init__(self, dims, rank, size, *, wdtype=0, layer_id=0, seed=0, bias=None,
                 routed_scale=1.0):
        self.d, self.r, self.R = dims, rank, size
        self.kw = dict(wdtype=wdtype, layer_id=layer_id, seed=seed)
        self.bias, self.routed_scale = bias, routed_scale
        self.qkv = None
        self.h1 = None

    def attn_partial(self, hidden, attn):
        x = hidden.numpy()
        self.qkv = otp.qkv_shard(self.d, x, self.r, self.R, **self.kw)
        return torch.from_numpy(otp.oproj_partial(self.d, attn.numpy(), self.r, self.R, **self.kw))

    def router_shard(self, hidden, p_sum):
        self.h1 = hidden.numpy() + p_sum.numpy()
        return torch.from_numpy(otp.router_shard(self.d, self.h1, self.r, self.R, bias=self.bias,
                                                 **self.kw))

    def moe_partial(self, logits):
        self.idx, self.gates = otp.select(logits.numpy(), self.d.top_k)
        return torch.from_numpy(otp.moe_partial(self.d, self.h1, self.idx, self.gates, self.r,
                                                self.R, routed_scale=self.routed_scale, **self.kw))

    def combine(self, y_sum, hidden):
        hidden.copy_(torch.from_numpy(self.h1 + y_sum.numpy()))
