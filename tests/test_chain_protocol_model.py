"""A model of the planned dependency-chained decode kernel's synchronisation,
checked on CPU before any GPU run.

The kernel (one persistent CTA per SM, all co-resident) runs the decoder's
linears as phases ({q,k,v}, {o}, {gate,up}, {down} per layer).  Between
phases each CTA
1. issues the next phase's weight copies (weights do not depend on
   activations),
2. writes its outputs of the phase, then increments a global counter
   (release),
3. waits, bounded, until the counter reaches G * (phase + 1) (acquire), or an
   abort flag is set; a wait that runs past its limit sets the abort flag and
   the TIMEOUT status,
4. reads the phase's input (all CTAs' outputs of the previous phase).

The model runs G CTAs in random interleavings with random work times, with
and without one CTA that never arrives (a stuck copy).  Checks:
- every CTA finishes (no hang);
- no CTA reads a phase's input before every CTA has written its part of it;
- TIMEOUT is raised exactly when an arrival was withheld, and then every CTA
  stops within one wait limit of the stall.
A planted mistake (increment before writing the outputs) must be caught.
"""
import random

import pytest

_ARRIVE_BEFORE_WRITE = False   # planted mistake, switched on by one test


class Chain:
    def __init__(self, ctas, phases, limit, withhold=None, seed=0):
        self.G, self.P, self.limit = ctas, phases, limit
        self.rng = random.Random(seed)
        self.counter = 0
        self.abort = False
        self.timeout = False
        self.written = [set() for _ in range(phases)]   # CTAs whose outputs of phase p are in memory
        self.withhold = withhold                        # (cta, phase) that never arrives
        self.bad_read = None
        self.clock = 0

    def cta(self, c):
        """Generator: one CTA, yielding once per step of simulated time."""
        for p in range(self.P):
            if p > 0:
                # acquire: wait for every CTA's arrival of phase p - 1
                waited = 0
                while self.counter < self.G * p and not self.abort:
                    waited += 1
                    if waited > self.limit:
                        self.abort = True
                        self.timeout = True
                        break
                    yield
                if self.abort:
                    return
                # read the phase's input: every CTA's outputs of phase p - 1
                if len(self.written[p - 1]) != self.G and self.bad_read is None:
                    self.bad_read = (c, p)
            # compute this CTA's share of phase p (random time), then publish
            for _ in range(self.rng.randint(1, 6)):
                yield
            if (c, p) == self.withhold:
                while not self.abort:      # stuck copy: never arrives, leaves when told to abort
                    yield
                return
            if _ARRIVE_BEFORE_WRITE:
                self.counter += 1
                yield                      # another CTA may run between the two
                self.written[p].add(c)
            else:
                self.written[p].add(c)
                self.counter += 1          # release after the writes

    def run(self, max_steps=100000):
        live = {c: self.cta(c) for c in range(self.G)}
        steps = 0
        while live:
            c = self.rng.choice(list(live))
            try:
                next(live[c])
            except StopIteration:
                del live[c]
            steps += 1
            if steps > max_steps:
                raise AssertionError("hang: CTAs still live after %d steps" % max_steps)
        return steps


@pytest.mark.parametrize("seed", range(40))
def test_chain_completes_and_never_reads_early(seed):
    ch = Chain(ctas=8, phases=12, limit=400, seed=seed)
    ch.run()
    assert not ch.timeout and not ch.abort
    assert ch.bad_read is None
    assert ch.counter == 8 * 12
    assert all(len(w) == 8 for w in ch.written)


@pytest.mark.parametrize("seed", range(20))
def test_withheld_arrival_times_out_everywhere_without_hanging(seed):
    rng = random.Random(1000 + seed)
    stuck = (rng.randrange(8), rng.randrange(11))
    ch = Chain(ctas=8, phases=12, limit=300, withhold=stuck, seed=seed)
    ch.run()
    assert ch.timeout and ch.abort
    assert ch.bad_read is None
    # nothing past the stuck phase was published by anyone
    assert all(len(w) == 0 for w in ch.written[stuck[1] + 1:])


def test_planted_arrive_before_write_is_caught():
    global _ARRIVE_BEFORE_WRITE
    _ARRIVE_BEFORE_WRITE = True
    try:
        caught = 0
        for seed in range(30):
            ch = Chain(ctas=8, phases=12, limit=400, seed=seed)
            ch.run()
            caught += ch.bad_read is not None
        assert caught > 0
    finally:
        _ARRIVE_BEFORE_WRITE = False
