"""Model check of the streaming router's end-of-tile protocol (CPU only).

After streaming its tile, each of the router's 8 compute warps
(router_stream_kernel):
  1. waits part_free (the previous tile's parts read), writes its parts,
     arrives on part_ready and waits for it;
  2. publishes its uncertain tokens (an atomic add on nunc, then their rows),
     arrives on unc_ready and waits for it, then reads nunc;
  3. for each batch of kUB uncertain tokens: writes its float64 partial
     logits of every token of the batch into p64, arrives on p64_ready and
     waits for it; the owner lanes then read all 8 warps' partials; unless it
     was the last batch, the warp arrives on p64_free and waits for it;
  4. decides its tokens, adds 1 to `done`; the warp that brings `done` to 8
     resets done and nunc; every warp arrives on part_free.
Every barrier counts 8 arrivals, phases taken from per-warp counters (the
tile index for part_ready and unc_ready, running phase bits for p64_ready and
p64_free). The model runs the 8 warps under random interleavings for several
tiles with random uncertain counts and checks that
  * every warp reads the tile's whole nunc (all publications before any read),
  * every owner reads 8 partials of its own batch (none stale, none of the
    next batch),
  * no warp writes a tile's parts before every warp has read the previous
    tile's, and nothing deadlocks.
Two broken schedules are caught: no p64_free barrier between batches (a fast
warp overwrites partials an owner has not read), and nunc reset by each warp
right after its own read (a slow warp reads a reset count).
"""
import random

import pytest
from test_pair_protocol_model import Bar

W, KUB = 8, 4


def simulate(unsure, seed, variant="shipped"):
    """unsure[t][h]: uncertain tokens warp h publishes in tile t."""
    rng = random.Random(seed)
    part_ready, part_free = Bar(W), Bar(W)
    unc_ready, p64_ready, p64_free = Bar(W), Bar(W), Bar(W)
    st = dict(nunc=0, done=0, parts=[None] * W, p64=[[None] * W for _ in range(KUB)])

    def warp(h):
        p64_phase = p64_free_phase = 0
        for it, counts in enumerate(unsure):
            # parts of this tile
            if it > 0:
                while not part_free.try_wait((it - 1) & 1):
                    yield False
            for hh in range(W):
                assert st["parts"][hh] in (None, it - 1, it), "parts overwritten too early"
            st["parts"][h] = it
            part_ready.arrive()
            while not part_ready.try_wait(it & 1):
                yield False
            for hh in range(W):
                assert st["parts"][hh] == it, f"warp {h} read stale parts of warp {hh}"
            yield True
            # publish, then read the tile's count
            st["nunc"] += counts[h]
            unc_ready.arrive()
            while not unc_ready.try_wait(it & 1):
                yield False
            nunc = st["nunc"]
            assert nunc == sum(counts), f"warp {h} read nunc {nunc}, tile {it} has {sum(counts)}"
            if variant == "reset_early":
                st["nunc"] = 0
            yield True
            nb_total = -(-nunc // KUB)
            for b in range(nb_total):
                nb = min(KUB, nunc - b * KUB)
                for u in range(nb):
                    st["p64"][u][h] = (it, b)
                    yield True
                p64_ready.arrive()
                while not p64_ready.try_wait(p64_phase):
                    yield False
                p64_phase ^= 1
                for u in range(nb):  # this warp's owner lanes of the batch, if any
                    for hh in range(W):
                        assert st["p64"][u][hh] == (it, b), \
                            f"owner in warp {h} read {st['p64'][u][hh]} for {(it, b)}"
                    yield True
                if b + 1 < nb_total and variant != "no_p64_free":
                    p64_free.arrive()
                    while not p64_free.try_wait(p64_free_phase):
                        yield False
                    p64_free_phase ^= 1
            # decisions; the last warp resets the counters
            st["done"] += 1
            if st["done"] == W:
                st["done"] = 0
                if variant != "reset_early":
                    st["nunc"] = 0
            part_free.arrive()
            yield True

    roles = [warp(h) for h in range(W)]
    idle = 0
    while roles:
        g = rng.choice(roles)
        try:
            idle = 0 if next(g) else idle + 1
        except StopIteration:
            roles.remove(g)
            idle = 0
        except AssertionError as ex:
            return f"stale: {ex}"
        if idle > 400 * len(roles):
            return "deadlock"
    return "ok"


def tiles_of(seed, ntiles):
    rng = random.Random(1000 + seed)
    out = []
    for _ in range(ntiles):
        # mostly none, sometimes a few, sometimes whole warps' worth (exact ties)
        kind = rng.random()
        out.append([rng.choice([0, 0, 0, 1]) if kind < 0.6 else
                    rng.randrange(0, 17) for _ in range(W)])
    return out


@pytest.mark.parametrize("ntiles", [1, 2, 5])
def test_shipped_fallback_protocol_survives_random_interleavings(ntiles):
    for seed in range(40):
        assert simulate(tiles_of(seed, ntiles), seed) == "ok", seed


def test_every_token_uncertain_runs_all_batches():
    # W_r = 0: every token of every tile is re-decided (32 batches per tile)
    for seed in range(5):
        assert simulate([[16] * W for _ in range(3)], seed) == "ok"


@pytest.mark.parametrize("variant", ["no_p64_free", "reset_early"])
def test_broken_fallback_schedules_are_caught(variant):
    results = [simulate([[rng_c for rng_c in random.Random(s).choices(range(0, 9), k=W)]
                         for _ in range(3)], s, variant) for s in range(60)]
    assert any(r.startswith("stale") for r in results), (variant, set(results))
