"""A host model of the OSK kernel's early-break protocol (max_run = r), checked under
random interleavings of the two softmax warpgroups.

Each warpgroup takes the groups of its parity in order.  A group's first vote is
taken against a stale running max, so it may send a group with no kept page to the
exact path, but never lets a group the exact vote keeps settle as all-skipped.  The
skip path settles at once; the exact path waits until the previous group is settled
(or gives up once its own group lies past the stop), then decides page by page from
the list position of the last kept page.  Any leader that can prove the break from
settled groups lowers the stop group index; a warpgroup stops at the first group at
or past it.

Checked: every processed page's decision equals the pages' rule cut at the break
(a page with r skipped pages right before it, and all later pages, skipped), every
page of a group no warpgroup reached lies past the break, and some warpgroup can
always move until both are done."""
import random

import pytest


def expected(keep_rule, r):
    out, last = [], -1
    for p, k in enumerate(keep_rule):
        if p - last - 1 >= r:
            out.extend([False] * (len(keep_rule) - p))
            break
        out.append(k)
        if k:
            last = p
    return out


def run(keep_rule, GP, r, seed):
    rng = random.Random(seed)
    n = len(keep_rule)
    ng = (n + GP - 1) // GP
    pages = lambda g: range(g * GP, min(n, g * GP + GP))
    stop = ng
    kept_last = -1
    settled = [-1, -1]           # last settled group per warpgroup
    decided = {}
    nxt = [0, 1]                 # next group per warpgroup
    phase = ["top", "top"]       # where each warpgroup is within its group
    done = [False, False]

    def all_before_settled(g, wg):
        return g == 0 or settled[wg ^ 1] >= g - 1

    def detect(g):
        nonlocal stop
        if (g + 1) * GP - kept_last - 1 >= r:
            stop = min(stop, g + 1)

    steps = 0
    while not all(done):
        steps += 1
        assert steps < 100000
        movable = []
        for wg in (0, 1):
            if done[wg]:
                continue
            g = nxt[wg]
            if phase[wg] == "exact_wait" and not (all_before_settled(g, wg) or g >= stop):
                continue
            movable.append(wg)
        assert movable, "no warpgroup can move"
        wg = rng.choice(movable)
        g = nxt[wg]
        if phase[wg] == "top":
            if g >= ng or g >= stop:
                done[wg] = True
                continue
            rule_keeps = any(keep_rule[p] for p in pages(g)) or g == 0
            # first vote: all-skip only when no page is kept by the exact rule
            phase[wg] = "exact_wait" if rule_keeps or rng.random() < 0.4 else "skip"
        elif phase[wg] == "skip":
            for p in pages(g):
                decided[p] = False
            if all_before_settled(g, wg):
                detect(g)
            settled[wg] = g
            nxt[wg] += 2
            phase[wg] = "top"
        else:  # exact path, its wait over
            if not all_before_settled(g, wg):   # gave up: the group lies past the stop
                assert g >= stop
                for p in pages(g):
                    decided[p] = False
            else:
                kl = kept_last
                past = False
                for p in pages(g):
                    past = past or p - kl - 1 >= r
                    k = (keep_rule[p] or p == 0) and not past
                    decided[p] = k
                    if k:
                        kl = p
                kept_last = kl
                detect(g)
            settled[wg] = g
            nxt[wg] += 2
            phase[wg] = "top"
    want = expected([k or p == 0 for p, k in enumerate(keep_rule)], r)
    for p in range(n):
        if p in decided:
            assert decided[p] == want[p], f"page {p}"
        else:
            assert p >= stop * GP and not want[p], f"page {p} not reached but not past the break"
    return stop < ng


@pytest.mark.parametrize("GP", [1, 2])
@pytest.mark.parametrize("r", [1, 2, 3, 8])
def test_early_break_protocol(GP, r):
    rng = random.Random(100 * GP + r)
    stopped = 0
    for seed in range(400):
        n = rng.randint(1, 60)
        density = rng.choice([0.05, 0.2, 0.5])
        keep_rule = [p == 0 or rng.random() < density for p in range(n)]
        stopped += run(keep_rule, GP, r, seed)
    assert stopped > 0  # the stop index did end lists early
