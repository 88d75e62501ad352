"""A host model of the OSK kernel's S-buffer hand-offs, checked under random
interleavings: QK^T issuers, in-order completion of each issuer's MMAs, and the
two softmax warpgroups.

An mbarrier wait names a phase only by its parity, so it passes whenever the
barrier's current phase has the other parity: correct if the wanted phase just
completed, wrong if the barrier has not yet completed the phase before it (the
waiter is ahead).  The model tracks the true events and flags any wait that
passes before the event it stands for, and a state where no thread can move.
It shows why the kernel keeps the S-buffer barriers per group parity once two
threads issue QK^T: with shared barriers such a wait does pass early, after
which the phases are out of step and the threads stall (the kernel's bounded
waits then time out); with per-parity barriers, and with a single issuer on
shared barriers, neither happens."""
import random

import pytest

SBG = 3  # S buffers


class Barrier:
    """Completed-phase counter with parity waits (arrival count 1)."""

    def __init__(self):
        self.done = 0

    def passes(self, phase: int) -> bool:
        return (self.done & 1) != (phase & 1)

    def arrive(self):
        self.done += 1


def run(n_groups: int, two_issuers: bool, per_parity: bool, seed: int) -> int:
    """Number of waits that passed before their event (0 = the protocol holds)."""
    rng = random.Random(seed)
    if per_parity:
        sfull = {(b, p): Barrier() for b in range(SBG) for p in range(2)}
        sfree = {(b, p): Barrier() for b in range(SBG) for p in range(2)}
        full_of = lambda g: (sfull[(g % SBG, g % 2)], g // (2 * SBG))
        free_wait = lambda g: (sfree[(g % SBG, g % 2)], (g - SBG) // (2 * SBG))
        free_arrive = lambda g: sfree[(g % SBG, (g + 1) % 2)]
    else:
        sfull = {b: Barrier() for b in range(SBG)}
        sfree = {b: Barrier() for b in range(SBG)}
        full_of = lambda g: (sfull[g % SBG], g // SBG)
        free_wait = lambda g: (sfree[g % SBG], g // SBG - 1)
        free_arrive = lambda g: sfree[g % SBG]
    issuers = [list(range(p, n_groups, 2)) for p in range(2)] if two_issuers else \
        [list(range(n_groups))]
    softmax = [list(range(w, n_groups, 2)) for w in range(2)]
    in_flight = [[] for _ in issuers]  # issued, not complete, in each issuer's order
    complete, released = set(), set()
    early = 0
    while any(issuers) or any(in_flight) or any(softmax):
        moves = []
        for i, q in enumerate(issuers):
            if q:
                g = q[0]
                if g < SBG:
                    moves.append(("issue", i, g, True))
                else:
                    bar, ph = free_wait(g)
                    if bar.passes(ph):
                        moves.append(("issue", i, g, (g - SBG) in released))
        for i, q in enumerate(in_flight):
            if q:
                moves.append(("complete", i, q[0], True))
        for w, q in enumerate(softmax):
            if q:
                bar, ph = full_of(q[0])
                if bar.passes(ph):
                    moves.append(("release", w, q[0], q[0] in complete))
        if not moves:
            return early + 1000  # no thread can move: a wait aliased behind
        kind, i, g, truly = rng.choice(moves)
        early += 0 if truly else 1
        if kind == "issue":
            issuers[i].pop(0)
            in_flight[i].append(g)
        elif kind == "complete":
            in_flight[i].pop(0)
            complete.add(g)
            full_of(g)[0].arrive()
        else:
            softmax[i].pop(0)
            released.add(g)
            free_arrive(g).arrive()
    return early


@pytest.mark.parametrize("per_parity", [True, False])
def test_single_issuer_never_passes_early(per_parity):
    assert all(run(40, False, per_parity, s) == 0 for s in range(300))


def test_two_issuers_with_per_parity_barriers_never_pass_early():
    assert all(run(40, True, True, s) == 0 for s in range(600))


def test_two_issuers_with_shared_barriers_can_pass_early():
    assert any(run(40, True, False, s) > 0 for s in range(600))
