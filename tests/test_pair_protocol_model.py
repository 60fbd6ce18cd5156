"""Model check of the SM-pair weight-gradient pipeline protocol (CPU only).

The SM-pair backward kernel (tc_bwd_pair_kernel, weight-gradient mode) feeds
one MMA issuer in CTA 0 from the shared-memory rings of two CTAs. Full K
blocks complete on CTA 0's full[s] barrier (both CTAs' TMA loads); the ragged
last K block of an expert completes on each CTA's own[s], where a fix-up warp
zeroes the rows past the expert's end before both report to CTA 0's ready[s].

This model gives mbarriers their PTX semantics (arrival count, transaction
count, and a parity wait that also succeeds for the phase before the current
one) and runs the roles -- two producers, two fix-up warps, the MMA issuer --
plus the asynchronous TMA completions and MMA commits under random
interleavings. It checks that the MMA only reads a stage holding the current
use's data in both CTAs (zeroed tail included) and that nothing deadlocks.
The same check on the earlier schedule, where CTA 0's fix-up warp waited on
full[s] with the ring phase, finds the stale read that schedule allowed.
"""
import random

import pytest


class Bar:
    """mbarrier: pending arrivals, transaction count, completed-phase count."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.done = count, count, 0, 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        assert self.pending >= 0
        self._complete()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending, self.tx = self.count, 0

    def try_wait(self, parity):
        # complete unless `parity` is the parity of the current, open phase
        return (self.done & 1) != parity


def simulate(uses, seed, schedule, stages=6):
    """uses: per K-block use, True when it is an expert's ragged last block."""
    rng = random.Random(seed)
    n = len(uses)
    cta = [dict(full=[Bar(1) for _ in range(stages)], own=[Bar(1) for _ in range(stages)],
                ready=[Bar(2) for _ in range(stages)], empty=[Bar(1) for _ in range(stages)],
                data=[None] * stages, zeroed=[None] * stages) for _ in range(2)]
    pending = []  # asynchronous completions (TMA landings, MMA commits)

    def producer(r):
        for u in range(n):
            st, ring = u % stages, (u // stages) & 1
            while not cta[r]["empty"][st].try_wait(ring ^ 1):
                yield
            ragged = uses[u]
            if schedule == "shipped":
                target = cta[r]["own"][st] if ragged else cta[0]["full"][st]
            else:  # earlier: ragged loads on each CTA's full[s]
                target = cta[r]["full"][st] if ragged else cta[0]["full"][st]
            if ragged:
                target.arrive(32)
            elif r == 0:
                target.arrive(64)

            def land(r=r, st=st, u=u, target=target):
                cta[r]["data"][st], cta[r]["zeroed"][st] = u, None
                target.complete_tx(32)
            pending.append(land)
            yield

    def fixup(r):
        own_par = 0
        for u in range(n):
            st, ring = u % stages, (u // stages) & 1
            if uses[u]:
                if schedule == "shipped":
                    bar, par = cta[r]["own"][st], (own_par >> st) & 1
                    own_par ^= 1 << st
                elif r == 0:
                    bar, par = cta[0]["full"][st], ring
                else:
                    bar, par = cta[1]["full"][st], (own_par >> st) & 1
                    own_par ^= 1 << st
                while not bar.try_wait(par):
                    yield
                assert cta[r]["data"][st] == u, f"fix-up of CTA {r} saw stale stage data"
                cta[r]["zeroed"][st] = u
                cta[0]["ready"][st].arrive()
            yield

    def mma():
        ready_par = full_par = 0
        for u in range(n):
            st, ring = u % stages, (u // stages) & 1
            if uses[u]:
                bar, par = cta[0]["ready"][st], (ready_par >> st) & 1
                ready_par ^= 1 << st
            else:
                bar = cta[0]["full"][st]
                if schedule == "shipped":
                    par = (full_par >> st) & 1
                    full_par ^= 1 << st
                else:
                    par = ring
            while not bar.try_wait(par):
                yield
            for r in range(2):
                assert cta[r]["data"][st] == u, f"MMA read stale data of CTA {r}"
                if uses[u]:
                    assert cta[r]["zeroed"][st] == u, f"MMA read an unzeroed tail of CTA {r}"

            def commit(st=st):
                for r in range(2):
                    cta[r]["empty"][st].arrive()
            pending.append(commit)
            yield

    roles = [producer(0), producer(1), fixup(0), fixup(1), mma()]
    for _ in range(2_000_000):
        if not roles and not pending:
            return "ok"
        if pending and (not roles or rng.random() < 0.3):
            pending.pop(rng.randrange(len(pending)))()
            continue
        g = rng.choice(roles)
        try:
            next(g)
        except StopIteration:
            roles.remove(g)
        except AssertionError as ex:
            return f"stale: {ex}"
    return "deadlock"


def random_uses(rng):
    kb = rng.choice([1, 2, 3, 5, 7, 13, 64])
    uses = []
    for _ in range(rng.choice([3, 10, 25])):
        uses += [False] * (kb - 1) + [rng.random() < 0.8]
    return uses


def test_shipped_schedule_survives_random_interleavings():
    for seed in range(120):
        uses = random_uses(random.Random(1000 + seed))
        assert simulate(uses, seed, "shipped") == "ok", seed


def test_earlier_schedule_is_caught():
    results = [simulate(random_uses(random.Random(1000 + seed)), seed, "earlier")
               for seed in range(60)]
    assert any(r.startswith("stale") for r in results)


@pytest.mark.parametrize("kb", [1, 64])
def test_all_ragged_and_no_ragged_sequences(kb):
    for ragged in (False, True):
        uses = ([False] * (kb - 1) + [ragged]) * 12
        for seed in range(10):
            assert simulate(uses, seed, "shipped") == "ok"
