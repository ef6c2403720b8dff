"""The stage ring's synchronisation, modelled on the CPU.

The attention kernels stream K/V tiles through a ring of shared-memory
stages: one producer fills tile t into stage t mod STAGES (an mbarrier whose
phase completes when the copy lands, in any order across stages); consumer
warp t mod NTW waits for the fill, reads the stage and releases it (a second
mbarrier the producer waits on before the stage's next fill).  A wait on an
mbarrier tests a phase *parity*: it succeeds when the barrier's phase in
progress has the other parity.

This model plays that protocol under random interleavings (copy completion
order, warp speeds) and checks what each warp reads.  It pins the argument
behind the kernels' waits:
  * parity alone is sound when STAGES is a multiple of NTW (each stage has one
    consumer warp, which cannot be a lap ahead of the stage's previous fill);
  * parity alone is NOT sound otherwise (13 stages, 4 warps): a fast warp can
    pass the parity test on the phase of the fill before the previous one;
  * the fill ticket (the producer stores the tile index before the fill, a
    warp first waits for its own index, then tests the parity) is sound for
    any stage count.
"""
import random

import pytest


def simulate(stages, ntw, n_tiles, ticket, seed, max_steps=200_000):
    """Play one random schedule; return the list of (tile wanted, tile read)
    mismatches, plus "stuck" if the schedule stopped making progress (which
    only a stale read leads to).  Actors: the producer, each consumer warp,
    and the copy engine landing any issued fill."""
    rng = random.Random(seed)
    full_done = [0] * stages      # completed phases of each stage's fill barrier
    empty_done = [0] * stages     # completed phases of each stage's release barrier
    content = [None] * stages     # tile whose bytes the stage holds (after landing)
    tick = [-1] * stages          # fill ticket
    in_flight = {}                # stage -> tile being copied (issued, not landed)
    next_fill = 0                 # producer: next tile to fill
    warp_next = list(range(ntw))  # each warp's next tile
    warp_busy = [0] * ntw         # steps of "math" left before the warp looks again
    errors = []

    def parity_ok(done, want_phase):
        # try_wait.parity(want_phase & 1): true when the phase in progress
        # (index `done`) has the other parity.
        return (done & 1) != (want_phase & 1)

    steps = 0
    while min(warp_next) < n_tiles:
        steps += 1
        if steps > max_steps:
            return errors + ["stuck"]
        actors = []
        if next_fill < n_tiles:
            s = next_fill % stages
            f = next_fill // stages
            # The producer may fill once the stage's previous fill was released
            # (its own waits are sound: it fills in order).
            if f == 0 or empty_done[s] >= f:
                if s not in in_flight:
                    actors.append("produce")
        if in_flight:
            actors.append("land")
        for w in range(ntw):
            if warp_next[w] < n_tiles:
                actors.append(("warp", w))
        a = rng.choice(actors)
        if a == "produce":
            s = next_fill % stages
            tick[s] = next_fill
            in_flight[s] = next_fill
            next_fill += 1
        elif a == "land":
            s = rng.choice(sorted(in_flight))
            content[s] = in_flight.pop(s)
            full_done[s] += 1
        else:
            w = a[1]
            if warp_busy[w]:
                warp_busy[w] -= 1
                continue
            t = warp_next[w]
            s, f = t % stages, t // stages
            ready = parity_ok(full_done[s], f)
            if ticket:
                ready = tick[s] == t and ready
            if not ready:
                continue
            if content[s] != t:
                errors.append((t, content[s]))
            empty_done[s] += 1           # release
            warp_next[w] += ntw
            warp_busy[w] = rng.choice([0, 0, 1, 3, 8])
    return errors


@pytest.mark.parametrize("stages,ntw", [(12, 4), (8, 4), (10, 5), (21, 7)])
def test_parity_alone_is_sound_with_whole_rounds(stages, ntw):
    for seed in range(60):
        assert simulate(stages, ntw, 200, ticket=False, seed=seed) == []


def test_parity_alone_fails_with_a_partial_round():
    bad = sum(bool(simulate(13, 4, 200, ticket=False, seed=seed)) for seed in range(200))
    assert bad > 0, "the model should reproduce the stale-phase read"


@pytest.mark.parametrize("stages,ntw", [(13, 4), (12, 4), (9, 4), (5, 4), (11, 7)])
def test_fill_ticket_is_sound_for_any_stage_count(stages, ntw):
    for seed in range(200):
        assert simulate(stages, ntw, 200, ticket=True, seed=seed) == []
