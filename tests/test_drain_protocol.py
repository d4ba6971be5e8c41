"""CPU model of how the tensor-bound LM head's 2-CTA pairs drain their copies
after giving up (no GPU).

Both CTAs of a pair load into the same ring of `S` stages; every copy
completes on the leader's barrier of its stage.  An mbarrier phase completes
when its arrival count reaches zero and its transaction count is zero; the
leader's producer makes the phase's one arrival with the bytes of both CTAs
(arrive.expect_tx), each landed copy subtracts its bytes (complete_tx), and
the count may go below zero while a copy lands before the arrival.  A stage
is refilled only after the consumer has waited on its phase, so one CTA runs
at most a ring ahead of the other.

After an abort at a random point, with copies still in flight, the leader
applies the fix-ups of lmhead_kernel's drain: from the two issue counts, a
load only the leader issued has the other CTA's bytes counted as arrived, a
load only the other CTA issued gets the leader's arrival with that CTA's
bytes alone.  The model checks, over many random interleavings, that each
stage's last phase then completes, and never before the last copy into that
stage has landed -- the property that lets both CTAs exit with nothing in
flight."""
import random

import pytest

B = 32768           # bytes one CTA loads per stage


class Barrier:
    def __init__(self):
        self.phase, self.pending, self.tx = 0, 1, 0

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending, self.tx = 1, 0

    def arrive_expect_tx(self, n):
        assert self.pending == 1
        self.pending -= 1
        self.tx += n
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        self._check()


def run(seed, S, tiles_k):
    rng = random.Random(seed)
    total = tiles_k                      # stage loads each CTA would issue without an abort
    bars = [Barrier() for _ in range(S)]
    issued = {"L": 0, "N": 0}
    consumed = 0                         # stage loads the consumer has waited on (in order)
    in_flight = []                       # (cta, load index) whose bytes have not landed
    landed = set()
    abort_at = rng.randrange(0, 4 * total + 1)
    steps = 0
    while steps < abort_at:
        steps += 1
        choice = rng.random()
        if choice < 0.3:                 # a producer issues its next load if its stage is free
            cta = rng.choice("LN")
            k = issued[cta]
            if k < total and k - S < consumed:        # stage k % S refilled only after load k - S was consumed
                if cta == "L":
                    bars[k % S].arrive_expect_tx(2 * B)
                in_flight.append((cta, k))
                issued[cta] += 1
        elif choice < 0.7 and in_flight:  # a copy lands
            cta, k = in_flight.pop(rng.randrange(len(in_flight)))
            bars[k % S].complete_tx(B)
            landed.add((cta, k))
        else:                            # the consumer takes the next full stage
            k = consumed
            if k < total and bars[k % S].phase > k // S:
                consumed += 1
    # abort: no more issues or consumption; the leader's fix-ups
    nL, nN = issued["L"], issued["N"]
    assert abs(nL - nN) <= S
    for k in range(min(nL, nN), max(nL, nN)):
        if nL > nN:
            bars[k % S].complete_tx(B)
        else:
            bars[k % S].arrive_expect_tx(B)
    n_all = max(nL, nN)

    def last_phase_done(q):
        k_last = q + ((n_all - 1 - q) // S) * S
        return bars[q].phase > k_last // S

    # remaining copies land in random order; a stage's last phase must not
    # complete while a copy into that stage is still in flight
    rng.shuffle(in_flight)
    for i, (cta, k) in enumerate(in_flight):
        for q in range(min(S, n_all)):
            if any(kk % S == q for _, kk in in_flight[i:]):
                assert not last_phase_done(q), (seed, q)
        bars[k % S].complete_tx(B)
    for q in range(min(S, n_all)):
        assert last_phase_done(q), (seed, q)
        # no phase ran past the loads issued into the stage
        assert bars[q].phase == (n_all - 1 - q) // S + 1
    return nL, nN


@pytest.mark.parametrize("S", [2, 4, 6])
def test_drain_completes_exactly_when_copies_land(S):
    seen_ahead = {"L": 0, "N": 0, "even": 0}
    for seed in range(1500):
        nL, nN = run(seed, S, tiles_k=3 * S + 5)
        seen_ahead["L" if nL > nN else ("N" if nN > nL else "even")] += 1
    # the random interleavings exercise both fix-ups and the balanced case
    assert min(seen_ahead.values()) > 20, seen_ahead
