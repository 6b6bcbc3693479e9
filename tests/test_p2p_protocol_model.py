"""A model of the one-kernel all-reduce's counter protocol, checked over random schedules.

The kernel (one cooperative launch per rank, C CTAs each) synchronises its three
phases through two monotonic counters per rank: every CTA adds 1 to its rank's
phase-1 counter after writing its part of the step-1 payloads, waits until every
rank's phase-1 counter reaches epoch * C, reads every rank's step-1 payloads,
writes its part of its rank's step-2 payload, adds 1 to the phase-2 counter,
waits for every rank's phase-2 counter to reach epoch * C, and reads every
owner's step-2 payload.  Calls of one rank run in stream order; calls of
different ranks overlap freely.  The epoch is either given (the k-th call passes
k) or derived by each CTA, before it counts, from its own rank's phase-1
counter: floor(read / C) + 1.

The model runs every CTA of every rank as a step machine under a random
scheduler and checks, at each read, that the data read is complete and belongs
to the same call (neither stale nor already overwritten by the next call), and
that a derived epoch equals the call's index.  It also shows the documented
hazard: a call that launches a different number of CTAs on the same counters
lets a wait pass early."""
import random

import pytest


class Violation(Exception):
    pass


class Model:
    def __init__(self, P, ctas, calls, seed, derived=True, bug=None, check_epoch=True):
        """ctas: CTAs per rank for each call (a list, one entry per call); bug: a planted
        protocol mistake (for checking that the model's checks catch it); check_epoch:
        also assert that a derived epoch equals the call's index (the kernel itself does
        not check it, so a test of what the kernel would read turns it off)."""
        self.P, self.ctas, self.calls, self.derived, self.bug = P, ctas, calls, derived, bug
        self.check_epoch = check_epoch
        self.rng = random.Random(seed)
        self.ctr1 = [0] * P
        self.ctr2 = [0] * P
        # version[p][i]: the call whose CTA i of rank p last wrote its part (0 = never)
        self.s1 = [dict() for _ in range(P)]
        self.s2 = [dict() for _ in range(P)]
        self.call_of = [0] * P          # the call each rank is running (stream order)
        self.live = [[] for _ in range(P)]

    def _cta(self, r, i, k, C):
        """Steps of CTA i of rank r in call k (1-based) with C CTAs per rank."""
        read = self.ctr1[r]
        epoch = read // C + (0 if self.bug == "epoch_off_by_one" else 1) if self.derived else k
        if self.check_epoch and self.derived and epoch != k:
            raise Violation(f"rank {r} CTA {i} call {k}: derived epoch {epoch}")
        yield
        self.s1[r][i] = k
        yield
        self.ctr1[r] += 1
        target = (epoch - 1 if self.bug == "target_one_call_behind" else epoch) * C
        while self.bug != "no_phase1_wait" and not all(c >= target for c in self.ctr1):
            yield "wait"
        for p in range(self.P):                      # reduce-scatter: read every rank's step-1 parts
            parts = self.s1[p]
            if len(parts) < C or any(v != k for v in parts.values()):
                raise Violation(f"rank {r} call {k} read step 1 of rank {p}: {sorted(parts.items())}")
        yield
        self.s2[r][i] = k
        yield
        self.ctr2[r] += 1
        while self.bug != "no_phase2_wait" and not all(c >= target for c in self.ctr2):
            yield "wait"
        for p in range(self.P):                      # all-gather: read every owner's step-2 parts
            parts = self.s2[p]
            if len(parts) < C or any(v != k for v in parts.values()):
                raise Violation(f"rank {r} call {k} read step 2 of rank {p}: {sorted(parts.items())}")
        yield

    def _launch(self, r):
        k = self.call_of[r] + 1
        if k > self.calls:
            return
        self.call_of[r] = k
        C = self.ctas[k - 1]
        self.live[r] = [self._cta(r, i, k, C) for i in range(C)]

    def run(self):
        for r in range(self.P):
            self._launch(r)
        while any(self.live):
            runnable = [(r, g) for r in range(self.P) for g in self.live[r]]
            self.rng.shuffle(runnable)
            progressed = False
            for r, g in runnable:
                try:
                    if next(g) != "wait":
                        progressed = True
                        break
                except StopIteration:
                    self.live[r].remove(g)
                    if not self.live[r]:
                        self._launch(r)      # the rank's next call starts when its kernel has ended
                    progressed = True
                    break
            if not progressed:
                raise Violation("no CTA can make progress")


@pytest.mark.parametrize("derived", [True, False], ids=["derived_epoch", "explicit_epoch"])
@pytest.mark.parametrize("P,C", [(2, 1), (2, 3), (4, 2), (8, 2), (3, 4)])
def test_protocol_holds_under_random_schedules(P, C, derived):
    for seed in range(60):
        Model(P, [C] * 5, 5, seed, derived).run()


def test_a_changed_cta_count_lets_a_wait_pass_early():
    """8 CTAs per rank in the first call, 3 in the second, on the same counters: the
    second call derives epoch floor(8/3) + 1 = 3 with target 9, which one count of
    that call already reaches, so some schedule reads step-1 data that is not
    complete -- what the kernel would do (no epoch self-check here)."""
    reads = 0
    for seed in range(200):
        try:
            Model(2, [8, 3], 2, seed, derived=True, check_epoch=False).run()
        except Violation as v:
            reads += "read step" in str(v)
    assert reads > 0


@pytest.mark.parametrize("bug", ["no_phase1_wait", "no_phase2_wait", "epoch_off_by_one", "target_one_call_behind"])
def test_the_model_catches_planted_protocol_mistakes(bug):
    """The model's data checks have teeth: each planted mistake in the protocol makes
    some schedule read incomplete or overwritten payloads (explicit epochs for the wait
    mistakes, derived for the epoch one; the epoch self-check is off)."""
    derived = bug == "epoch_off_by_one"
    reads = 0
    for seed in range(100):
        try:
            Model(2, [3] * 4, 4, seed, derived=derived, bug=bug, check_epoch=False).run()
        except Violation as v:
            reads += "read step" in str(v)
    assert reads > 0, bug
