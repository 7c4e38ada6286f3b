"""The single-launch decode kernel's grid-barrier protocol, checked as a
model on the CPU under adversarial schedules.

The kernel's barrier word (workspace header, 8 bytes) holds an arrival count
(low 32 bits) and an epoch (high 32 bits). Each CTA of a call reads the epoch
after the previous kernel has completed, adds its arrival (atomic), and then:
the arrival that brings the count to the grid size G then stores (epoch + 1,
count 0); every other CTA waits, with a time limit, until it sees the count at
G or an epoch that differs from the one it read, or gives up (the time
limit is checked before each poll). This model runs that protocol
step by step with random interleavings, CTAs that start only after others
have already given up, and random time limits, and checks that

* a CTA passes only after all G CTAs have arrived (or reports a timeout);
* with no time limit every CTA passes;
* after every call, whatever the schedule, the count is 0 and the epoch has
  advanced by exactly one, so the next call starts from a valid header.

It is a model of the protocol, not of the CUDA code; the GPU tests check the
kernel itself (tests/test_gpu_fused_decode.py).
"""
import random

import pytest

MASK = 0xFFFFFFFF


class Header:
    def __init__(self, arrive=0, epoch=0):
        self.arrive, self.epoch = arrive, epoch


def run_call(h, G, rng, limit=None, late=()):
    """One call of G CTAs; those in 'late' start only after the others have
    run for a while (each of them passed, gave up or is still waiting).
    Returns the sets of CTAs that passed and that gave up."""
    # per CTA: program counter 0 read epoch, 1 arrive, 2 wait, 3 done, 4 (the
    # last arrival only) store the new epoch and reset the count
    pc = [0] * G
    e0 = [None] * G
    waited = [0] * G
    arrived = set()
    passed_after_all = set()
    passed, timed_out = set(), set()
    early = [c for c in range(G) if c not in late]

    def step(c):
        if pc[c] == 0:
            e0[c] = h.epoch
            pc[c] = 1
        elif pc[c] == 1:
            ticket = h.arrive
            h.arrive = (h.arrive + 1) & MASK
            arrived.add(c)
            if ticket == G - 1:
                passed.add(c)
                passed_after_all.add(len(arrived) == G)
                pc[c] = 4
            else:
                pc[c] = 2
        elif pc[c] == 4:
            h.arrive, h.epoch = 0, (e0[c] + 1) & MASK
            pc[c] = 3
        elif pc[c] == 2:
            # the time limit is checked before each poll
            if limit is not None and waited[c] >= limit:
                timed_out.add(c)
                pc[c] = 3
            elif h.epoch != e0[c] or h.arrive >= G:
                passed.add(c)
                passed_after_all.add(len(arrived) == G)
                pc[c] = 3
            else:
                waited[c] += 1

    # the early CTAs run interleaved for a while (each passes, gives up or is
    # still waiting), then the late ones start and everything runs interleaved
    # until every CTA has passed or given up
    for _ in range(20 * G):
        live = [c for c in early if pc[c] != 3]
        if not live:
            break
        step(rng.choice(live))
    while any(pc[c] != 3 for c in range(G)):
        step(rng.choice([c for c in range(G) if pc[c] != 3]))
    assert passed_after_all <= {True}
    return passed, timed_out


@pytest.mark.parametrize("seed", range(20))
def test_every_cta_passes_without_a_limit(seed):
    rng = random.Random(seed)
    h = Header(0, rng.randrange(1 << 32))
    G = rng.randrange(1, 160)
    e = h.epoch
    passed, timed_out = run_call(h, G, rng)
    assert passed == set(range(G)) and not timed_out
    assert (h.arrive, h.epoch) == (0, (e + 1) & MASK)


@pytest.mark.parametrize("seed", range(40))
def test_header_valid_after_timeouts_and_late_ctas(seed):
    # random limits (including none and a single poll) and CTAs that start
    # after the others have given up: the header is valid after every call
    rng = random.Random(1000 + seed)
    h = Header(0, rng.randrange(1 << 32))
    for _ in range(6):
        G = rng.randrange(1, 64)
        late = set(rng.sample(range(G), rng.randrange(0, min(G, 4) + 1)))
        limit = rng.choice([None, 0, 1, 5, 50])
        e = h.epoch
        passed, timed_out = run_call(h, G, rng, limit=limit, late=late)
        assert passed | timed_out == set(range(G)) and not passed & timed_out
        assert (h.arrive, h.epoch) == (0, (e + 1) & MASK)
    # and a call with no limit afterwards passes everywhere
    G = 148
    passed, timed_out = run_call(h, G, rng)
    assert passed == set(range(G)) and not timed_out


def test_late_cta_reads_the_current_epoch():
    # every other CTA gave up before the last one even started: the last one
    # still reads the epoch the call began with (the epoch cannot change
    # before its own arrival), completes the count and resets it
    rng = random.Random(7)
    h = Header(0, 41)
    passed, timed_out = run_call(h, 8, rng, limit=0, late={5})
    assert timed_out == set(range(8)) - {5} and passed == {5}
    assert (h.arrive, h.epoch) == (0, 42)
