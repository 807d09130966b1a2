"""Progress of the one-read quantisation kernels' waits, on a model of the
schedule (host logic, no GPU).

The kernels hand out work items by ticket: a CTA takes the next ticket when it
starts, so tickets follow start order.  A (head, K|V) group's `tiles` items
hold consecutive tickets; an item publishes its partial statistics and then
waits until all items of its group have published.  The model runs CTAs on
R resident slots in random order and checks that every schedule completes when
a group fits in the resident set (tiles <= R; the launcher requires
2 tiles <= R), and that a schedule can deadlock when it does not, which is why
the launcher then takes the two-pass path.  Items that never wait (the Q tiles
folded in, or K tiles without smooth K) are modelled too.
"""
import random

import pytest


def run_schedule(groups, tiles, resident, rng, free_items=0):
    """Simulates ticketed CTAs; returns True if every CTA finished, False on deadlock.
    free_items: items per group position that never wait (placed after each group)."""
    per_group = tiles + free_items
    total = groups * per_group
    next_ticket = 0
    published = [0] * groups
    running = []  # [ticket, state]; state 0: loading, 1: published and waiting
    done = 0
    while done < total:
        # start CTAs while slots are free (each takes the next ticket)
        while len(running) < resident and next_ticket < total:
            running.append([next_ticket, 0])
            next_ticket += 1
        progress = False
        rng.shuffle(running)
        for cta in list(running):
            t, state = cta
            g, r = divmod(t, per_group)
            if r >= tiles:  # an item that never waits
                running.remove(cta)
                done += 1
                progress = True
            elif state == 0:  # tile loaded: publish
                published[g] += 1
                cta[1] = 1
                progress = True
            elif published[g] == tiles:  # the group is complete: encode and exit
                running.remove(cta)
                done += 1
                progress = True
        if not progress:
            return False
    return True


@pytest.mark.parametrize("tiles", [1, 2, 7, 32, 139, 256])
def test_every_schedule_completes_when_a_group_fits(tiles):
    rng = random.Random(tiles)
    for resident in (tiles, tiles + 1, 2 * tiles, 3 * tiles + 5):
        for free_items in (0, 3):
            for _ in range(5):
                assert run_schedule(groups=6, tiles=tiles, resident=resident, rng=rng, free_items=free_items)


@pytest.mark.parametrize("tiles", [2, 8, 33])
def test_a_group_larger_than_the_resident_set_deadlocks(tiles):
    # every resident CTA belongs to the first group and waits for tickets that cannot start
    assert not run_schedule(groups=2, tiles=tiles, resident=tiles - 1, rng=random.Random(0))


def test_launcher_margin():
    # the launcher takes the one-read path only when 2 tiles <= resident CTAs; the
    # prefill (32 tiles), long-GQA (256) and video (139) heads all fit the B200's
    # 148 SMs x 5 CTAs of the K/V kernel
    resident = 148 * 5
    for tiles in (32, 139, 256):
        assert 2 * tiles <= resident
        assert run_schedule(groups=4, tiles=tiles, resident=resident, rng=random.Random(tiles))
