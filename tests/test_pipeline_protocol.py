"""A model of the FP8 expert kernels' per-CTA pipeline (the roles and the
mbarrier phases they wait on by parity), run under every interleaving a
random scheduler picks, to check the rule the kernels follow: a converter
takes every n-th stage with n = min(converters, activation slots, stages),
which keeps each parity wait unambiguous.  The model reports a deadlock
(every role waiting) for a larger n and none with the rule.

Roles (one per kernel warp role): the weight producer (waits a free stage),
the copier (waits a free activation slot), the converters (per stage: the
slot's rows and the stage's B tile free), the MMA issuer (per unit: a free
accumulator; per stage: weights and B terms landed) and the epilogue (per
unit: the accumulator full).  An mbarrier completes a phase when its count
of arrivals is in; a wait on parity p passes while the current phase's
parity differs from p (the hardware's phase-parity rule)."""
import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passes(self, parity):
        return (self.phase & 1) != parity


def _run(units, nst, nxs, nconv_used, nconv_warps, seed):
    rng = random.Random(seed)
    full = [_Bar(1) for _ in range(nst)]
    empty = [_Bar(1) for _ in range(nst)]
    afull = [_Bar(1) for _ in range(nst)]
    xfull = [_Bar(1) for _ in range(nxs)]
    xempty = [_Bar(1) for _ in range(nxs)]
    accfull = [_Bar(1) for _ in range(2)]
    accempty = [_Bar(1) for _ in range(2)]

    def producer():
        it = 0
        for nkc in units:
            for _ in range(nkc):
                s = it % nst
                yield empty[s], ((it // nst) & 1) ^ 1
                afull[s].arrive()
                it += 1

    def copier():
        it = 0
        for nkc in units:
            for _ in range(nkc):
                x = it % nxs
                yield xempty[x], ((it // nxs) & 1) ^ 1
                xfull[x].arrive()
                it += 1

    def converter(cw):
        if cw >= nconv_used:
            return
        it = 0
        for nkc in units:
            for _ in range(nkc):
                if it % nconv_used == cw:
                    s, x = it % nst, it % nxs
                    yield xfull[x], (it // nxs) & 1
                    yield empty[s], ((it // nst) & 1) ^ 1
                    xempty[x].arrive()
                    full[s].arrive()
                it += 1

    def issuer():
        it = 0
        for nu, nkc in enumerate(units):
            b = nu & 1
            yield accempty[b], ((nu >> 1) & 1) ^ 1
            for _ in range(nkc):
                s, ph = it % nst, (it // nst) & 1
                yield afull[s], ph
                yield full[s], ph
                empty[s].arrive()     # the MMAs' commit
                it += 1
            accfull[b].arrive()

    def epilogue():
        for nu, _ in enumerate(units):
            b = nu & 1
            yield accfull[b], (nu >> 1) & 1
            accempty[b].arrive()

    roles = [producer(), copier(), issuer(), epilogue()] + [converter(c) for c in range(nconv_warps)]
    waits = []
    for r in roles:
        waits.append(next(r, None))
    while True:
        live = [i for i, w in enumerate(waits) if w is not None]
        if not live:
            return True
        ready = [i for i in live if waits[i][0].passes(waits[i][1])]
        if not ready:
            return False          # every live role waits: a deadlock
        i = rng.choice(ready)
        waits[i] = next(roles[i], None)


def _cases(seed):
    rng = random.Random(seed)
    for _ in range(25):
        units = [rng.randint(1, 56) for _ in range(rng.randint(1, 24))]
        nst, nxs, warps = rng.choice([2, 3, 5, 9]), rng.choice([2, 3, 5, 13, 16]), rng.choice([1, 2, 3, 4])
        yield units, nst, nxs, warps


def test_the_converter_rule_never_deadlocks():
    for case, (units, nst, nxs, warps) in enumerate(_cases(1)):
        n = min(warps, nxs, nst)
        for seed in range(4):
            assert _run(units, nst, nxs, n, warps, seed), (units, nst, nxs, warps)


def test_more_converters_than_slots_can_deadlock():
    """Three converters taking stages in turn over two activation slots: a
    converter two slot-fills behind reads the previous fill's phase as its
    own, runs ahead, and the pipeline stalls."""
    units = [56, 56, 56]
    assert any(not _run(units, 9, 2, 3, 3, seed) for seed in range(8))
    assert all(_run(units, 9, 2, 2, 3, seed) for seed in range(8))
