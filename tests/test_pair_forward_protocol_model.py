"""Model check of the SM-pair forward GEMM protocol (CPU only).

The forward grouped GEMM (tc_pair_gemm_kernel: Conv+Gate, Out, in-projection)
runs on a 2-CTA cluster. One MMA issuer in CTA 0 reads both CTAs' shared-
memory rings and writes both CTAs' TMEM accumulators (two buffers per CTA):
  full[s]   in CTA 0 only: CTA 0's producer arms it with both CTAs' bytes;
            the two TMA loads of each CTA (A rows, B rows) complete on it;
  empty[s]  one per CTA, both arrived by the MMA commit (multicast);
  tfull[a]  one per CTA, arrived by the commit after a tile's last MMA;
  tempty[a] in CTA 0 only, count 8: the four epilogue warps of each CTA
            (CTA 1's through the cluster window).
The model gives mbarriers their PTX semantics (arrival count, transaction
count that may run ahead of the arming arrival, a parity wait that also
passes for the phase before the current one), runs the roles -- two
producers, the MMA issuer, eight epilogue warps -- and the asynchronous TMA
landings and MMA commits under random interleavings, and checks that
  * every MMA reads the current use's data in both CTAs' stages,
  * no tile's MMAs start on an accumulator buffer that an epilogue warp of
    either CTA is still to read,
  * every epilogue warp reads its own tile's accumulator,
  * nothing deadlocks.
Two deliberately broken schedules are caught: tempty counting only CTA 0's
epilogue warps, and the MMA waiting on tempty with the unflipped phase.
"""
import random

import pytest
from test_pair_protocol_model import Bar

STAGES, LOAD_BYTES = 6, 16  # two loads (A, B) of LOAD_BYTES per CTA per stage


def simulate(tiles, kb, seed, variant="shipped"):
    rng = random.Random(seed)
    tempty_count = 4 if variant == "tempty_cta0_only" else 8
    full0 = [Bar(1) for _ in range(STAGES)]
    empty = [[Bar(1) for _ in range(STAGES)] for _ in range(2)]
    tfull = [[Bar(1) for _ in range(2)] for _ in range(2)]
    tempty0 = [Bar(tempty_count) for _ in range(2)]
    stage_data = [[None] * STAGES for _ in range(2)]   # use index held by each CTA's stage
    acc_tile = [[None] * 2 for _ in range(2)]          # tile held by each CTA's TMEM buffer
    epi_done = [[-1] * 4 for _ in range(2)]            # last tile read by each epilogue warp
    pending = []

    def producer(r):
        for u in range(tiles * kb):
            st, ring = u % STAGES, (u // STAGES) & 1
            while not empty[r][st].try_wait(ring ^ 1):
                yield False
            if r == 0:
                full0[st].arrive(2 * 2 * LOAD_BYTES)
            for _ in range(2):  # the A and B loads of this CTA
                def land(r=r, st=st, u=u):
                    stage_data[r][st] = u
                    full0[st].complete_tx(LOAD_BYTES)
                pending.append(land)
            yield True

    def mma():
        u = 0
        for t in range(tiles):
            a, ph = t & 1, (t >> 1) & 1
            par = ph if variant == "tempty_unflipped" else ph ^ 1
            while not tempty0[a].try_wait(par):
                yield False
            for r in range(2):
                for w in range(4):
                    assert epi_done[r][w] >= t - 2, \
                        f"tile {t} starts on buffer {a} before CTA {r} warp {w} read tile {t - 2}"
            for _ in range(kb):
                st, ring = u % STAGES, (u // STAGES) & 1
                while not full0[st].try_wait(ring):
                    yield False
                for r in range(2):
                    assert stage_data[r][st] == u, f"MMA read stale stage data of CTA {r}"

                def commit_stage(st=st):
                    for r in range(2):
                        empty[r][st].arrive()
                pending.append(commit_stage)
                u += 1
                yield True

            def commit_tile(a=a, t=t):
                for r in range(2):
                    acc_tile[r][a] = t
                    tfull[r][a].arrive()
            pending.append(commit_tile)
            yield True

    def epilogue(r, w):
        for t in range(tiles):
            a, ph = t & 1, (t >> 1) & 1
            while not tfull[r][a].try_wait(ph):
                yield False
            assert acc_tile[r][a] == t, f"CTA {r} warp {w} read tile {acc_tile[r][a]} for {t}"
            epi_done[r][w] = t
            if r == 0 or tempty_count == 8:
                tempty0[a].arrive()
            yield True

    roles = [producer(0), producer(1), mma()] + [epilogue(r, w) for r in range(2) for w in range(4)]
    idle = 0  # role steps in a row that found every wait still blocked
    while roles or pending:
        if pending and (not roles or rng.random() < 0.3):
            pending.pop(rng.randrange(len(pending)))()
            idle = 0
            continue
        g = rng.choice(roles)
        try:
            idle = 0 if next(g) else idle + 1
        except StopIteration:
            roles.remove(g)
            idle = 0
        except AssertionError as ex:
            return f"stale: {ex}"
        if idle > 200 * len(roles) and not pending:
            return "deadlock"
    return "ok"


@pytest.mark.parametrize("kb", [1, 2, 5, 16])
def test_shipped_forward_protocol_survives_random_interleavings(kb):
    for seed in range(30):
        tiles = random.Random(seed).choice([1, 2, 3, 7, 12])
        assert simulate(tiles, kb, seed) == "ok", (tiles, seed)


@pytest.mark.parametrize("variant,symptom", [("tempty_cta0_only", "stale"),
                                             ("tempty_unflipped", "deadlock")])
def test_broken_forward_schedules_are_caught(variant, symptom):
    results = [simulate(random.Random(seed).choice([3, 7, 12]), 2, seed, variant)
               for seed in range(60)]
    assert any(r.startswith(symptom) for r in results), (variant, set(results))
