"""A model of the router's selection as the kernels run it (one warp per
token, 32 lanes, `redux.sync` rounds on 32-bit keys; the per-expert lists
placed by 8 warps over contiguous code ranges), step for step in numpy, checked
against the definitions it must reproduce: the top-k by (value, then lower
expert id) and a stable sort of the (token, slot) codes by expert.  It pins
the algorithm's design on the CPU; the GPU tests compare the kernels
themselves with the oracle."""
import numpy as np
import pytest


def order_bits(v: np.float32) -> int:
    u = int(np.float32(v).view(np.uint32))
    if (u << 1) & 0xFFFFFFFF == 0:
        u = 0   # -0 ranks with +0
    return (~u) & 0xFFFFFFFF if u & 0x80000000 else u | 0x80000000


def topk_warp(keys_f32: np.ndarray, k: int) -> list:
    """The warp's rounds: each lane keeps its best remaining key (largest
    order bits, then lowest slot); a round takes the largest order bits over
    the lanes, then among the lanes holding them the largest complemented
    expert id; the owner lane drops it."""
    E = keys_f32.shape[0]
    per = -(-E // 32)
    hk = [[order_bits(keys_f32[l + 32 * q]) if l + 32 * q < E else 0 for q in range(per)]
          for l in range(32)]
    live = [[l + 32 * q < E for q in range(per)] for l in range(32)]

    def lane_best(l):
        bh, bq = 0, -1
        for q in range(per):
            if live[l][q] and (bq < 0 or hk[l][q] > bh):
                bh, bq = hk[l][q], q
        return bh, bq

    best = [lane_best(l) for l in range(32)]
    out = []
    for _ in range(k):
        bhi = max(b[0] for b in best)
        lo = [((~(l + 32 * b[1])) & 0xFFFFFFFF) if (b[1] >= 0 and b[0] == bhi) else 0
              for l, b in enumerate(best)]
        blo = max(lo)
        e = (~blo) & 0xFFFFFFFF
        owner = e & 31
        assert best[owner][0] == bhi and owner + 32 * best[owner][1] == e
        live[owner][best[owner][1]] = False
        best[owner] = lane_best(owner)
        out.append(e)
    return out


def place_codes(sel: np.ndarray, E: int, nwalk: int = 8) -> np.ndarray:
    """Counts per (warp range, expert), each warp's first place per expert,
    the expert offsets, then every code at offset + warp base + its rank
    among the earlier equal codes of its 32-code step + the step's running
    count."""
    ncode = sel.shape[0]
    span = ((ncode + nwalk - 1) // nwalk + 31) & ~31
    wc = np.zeros((nwalk, E), np.int64)
    for w in range(nwalk):
        for c in range(w * span, min(ncode, (w + 1) * span)):
            wc[w, sel[c]] += 1
    cnt = wc.sum(0)
    base = np.cumsum(wc, 0) - wc          # each warp's first place within the expert
    off = np.cumsum(cnt) - cnt
    perm = np.full(ncode, -1, np.int64)
    run = np.zeros((nwalk, E), np.int64)
    for w in range(nwalk):
        for c0 in range(w * span, min(ncode, (w + 1) * span), 32):
            step = list(range(c0, min(c0 + 32, min(ncode, (w + 1) * span))))
            for i, c in enumerate(step):
                rank = sum(1 for c2 in step[:i] if sel[c2] == sel[c])
                perm[off[sel[c]] + base[w, sel[c]] + run[w, sel[c]] + rank] = c
            for c in step:
                run[w, sel[c]] += 1
    return perm


@pytest.mark.parametrize("E,k", [(8, 2), (256, 8), (384, 8), (1000, 16)])
def test_topk_rounds_match_the_definition(E, k):
    rng = np.random.default_rng(E)
    for trial in range(6):
        v = rng.standard_normal(E).astype(np.float32)
        if trial % 2:                 # exact ties, and signed zeros
            v[rng.integers(0, E, E // 4)] = v[0]
            v[rng.integers(0, E, 3)] = np.float32(-0.0)
            v[rng.integers(0, E, 3)] = np.float32(0.0)
        key = (v.astype(np.float64), np.arange(E))
        want = sorted(range(E), key=lambda e: (-(key[0][e] + 0.0), e))[:k]
        assert topk_warp(v, k) == want


def test_topk_rounds_break_ties_to_the_lower_expert():
    v = np.zeros(64, np.float32)
    v[[40, 7, 33, 8]] = 1.0          # four equal largest values
    assert topk_warp(v, 3) == [7, 8, 33]


@pytest.mark.parametrize("M,k,E", [(1, 8, 256), (8, 8, 256), (33, 16, 640), (64, 16, 1024),
                                   (64, 8, 8)])
def test_code_placement_is_a_stable_sort_by_expert(M, k, E):
    rng = np.random.default_rng(M * 1000 + E)
    sel = np.stack([rng.choice(E, k, replace=False) for _ in range(M)]).reshape(-1)
    perm = place_codes(sel, E)
    assert np.array_equal(perm, np.argsort(sel, kind="stable"))
