"""Tensor-parallel slices of the decode layer, for the sharded path's tests --
TEST INFRASTRUCTURE ONLY (only tests/ imports this module).

The pages shard the layer over the GPUs of a node (wireai.ir "vLLM Blackwell
Kimi decode", section "4 key changes", items 2 and 3: the o-proj partial
sums are reduced across GPUs inside the receiving kernel together with the
residual, and the router scores are computed by the tensor-parallel ranks
among themselves).  These functions are the plain definitions of what one
rank of R computes, in fp64 from the same decoded weights as ``oracle.layer``
(one matrix product per step):

  q heads        rank r owns heads [r Hq/R, (r+1) Hq/R) and the kv heads they
                 read (head q reads kv head q div (Hq/Hkv)): QKV rows of those
                 heads, and o-proj input columns of its q heads
  o-proj         p_r = Wo[:, cols_r] a[:, cols_r];    h1 = x + sum_r p_r
  router         experts [r E/R, (r+1) E/R):  logits[:, E_r] = Wr[E_r] h1 (+ b)
  selection      on the gathered logits, identical on every rank
  experts        intermediate rows [r I/R, (r+1) I/R) of every expert (shared
                 and routed): y_r = shared_r(h1) + s sum_j g_j expert_{j,r}(h1),
                 expert_{e,r}(v) = Wd_e[:, I_r] (silu(Wg_e[I_r] v) * (Wu_e[I_r] v))
  output         out = h1 + sum_r y_r

Summing the R partial sums reproduces the unsharded layer up to the order of
additions (fp64: ~1e-15 relative).
"""
from __future__ import annotations

import numpy as np

from . import weight_rows


def span(n: int, rank: int, size: int) -> tuple[int, int]:
    """Rank's contiguous share [lo, hi) of n items (n divisible by size)."""
    if n % size:
        raise ValueError(f"{n} items do not split over {size} ranks")
    return n * rank // size, n * (rank + 1) // size


def kv_span(dims, rank: int, size: int) -> tuple[int, int]:
    """The kv heads the rank's q heads read."""
    q0, q1 = span(dims.q_heads, rank, size)
    grp = dims.q_heads // dims.kv_heads
    return q0 // grp, (q1 - 1) // grp + 1


def qkv_rows(dims, rank: int, size: int) -> np.ndarray:
    """Logical QKV output rows of the rank: its q heads, then k and v of its kv heads."""
    hd = dims.head_dim
    q0, q1 = span(dims.q_heads, rank, size)
    k0, k1 = kv_span(dims, rank, size)
    qo, ko, vo = 0, dims.q_heads * hd, (dims.q_heads + dims.kv_heads) * hd
    return np.concatenate([np.arange(qo + q0 * hd, qo + q1 * hd),
                           np.arange(ko + k0 * hd, ko + k1 * hd),
                           np.arange(vo + k0 * hd, vo + k1 * hd)])


def attn_cols(dims, rank: int, size: int) -> tuple[int, int]:
    q0, q1 = span(dims.q_heads, rank, size)
    return q0 * dims.head_dim, q1 * dims.head_dim


def _w(dims, kind, expert, row0, nrows, wdtype, layer_id, seed):
    return weight_rows(dims, kind, expert, row0, nrows, wdtype=wdtype, layer_id=layer_id, seed=seed)


def qkv_shard(dims, x, rank, size, *, wdtype=0, layer_id=0, seed=0):
    """qkv[:, qkv_rows(rank)] = x Wqkv[rows]^T."""
    rows = qkv_rows(dims, rank, size)
    W = np.stack([_w(dims, 1, 0, int(r), 1, wdtype, layer_id, seed)[0] for r in rows])
    return np.asarray(x, np.float64) @ W.T


def oproj_partial(dims, attn, rank, size, *, wdtype=0, layer_id=0, seed=0):
    """p_r = a[:, cols_r] Wo[:, cols_r]^T  [M, H]."""
    c0, c1 = attn_cols(dims, rank, size)
    Wo = _w(dims, 2, 0, 0, dims.hidden, wdtype, layer_id, seed)
    return np.asarray(attn, np.float64)[:, c0:c1] @ Wo[:, c0:c1].T


def router_shard(dims, h1, rank, size, *, bias=None, wdtype=0, layer_id=0, seed=0):
    """logits[:, E_r] = h1 Wr[E_r]^T (+ b[E_r])."""
    e0, e1 = span(dims.n_experts, rank, size)
    Wr = _w(dims, 3, 0, e0, e1 - e0, wdtype, layer_id, seed)
    lg = np.asarray(h1, np.float64) @ Wr.T
    if bias is not None:
        lg = lg + np.asarray(bias, np.float64)[e0:e1]
    return lg


def select(logits, k: int):
    """Top-k (ties to the lower expert id) and the softmax over the k selected
    logits, per token (the selection every rank makes on the gathered logits)."""
    logits = np.asarray(logits, np.float64)
    M, E = logits.shape
    idx = np.zeros((M, k), np.int32)
    gates = np.zeros((M, k))
    for t in range(M):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))[:k]
        idx[t] = order
        v = logits[t, order]
        w = np.exp(v - v.max())
        gates[t] = w / w.sum()
    return idx, gates


def _expert_slice(dims, e, h1, i0, i1, wdtype, layer_id, seed):
    n = i1 - i0
    Wg = _w(dims, 4, e, i0, n, wdtype, layer_id, seed)
    Wu = _w(dims, 5, e, i0, n, wdtype, layer_id, seed)
    Wd = _w(dims, 6, e, 0, dims.hidden, wdtype, layer_id, seed)[:, i0:i1]
    g = h1 @ Wg.T
    act = g / (1.0 + np.exp(-g)) * (h1 @ Wu.T)
    return act @ Wd.T


def moe_partial(dims, h1, idx, gates, rank, size, *, wdtype=0, layer_id=0, seed=0,
                routed_scale=1.0):
    """y_r = shared_r(h1) + s sum_j g_j expert_{idx_j, r}(h1)   [M, H]."""
    h1 = np.asarray(h1, np.float64)
    M = h1.shape[0]
    i0, i1 = span(dims.inter, rank, size)
    y = np.zeros((M, dims.hidden))
    if dims.n_shared:
        y += _expert_slice(dims, -1, h1, i0, i1, wdtype, layer_id, seed)
    cache = {}
    for t in range(M):
        routed = np.zeros(dims.hidden)
        for j in range(idx.shape[1]):
            e = int(idx[t, j])
            if e not in cache:
                cache[e] = _expert_slice(dims, e, h1, i0, i1, wdtype, layer_id, seed)
            routed += gates[t, j] * cache[e][t]
        y[t] += routed_scale * routed
    return y
