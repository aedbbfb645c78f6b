"""A randomised model of the in-kernel split merge's group protocol.

The n CTAs of a split group (one per chunk of a unit's K/V tiles) meet only
at one 64-bit word per group (arrivals in the high half, abandoned shares in
the low half) and a departure counter, so the protocol can be checked on the
CPU. This model runs n CTAs in random interleavings, with at most `slots` of
them resident at once (another kernel may hold the other SMs, so a group's
CTAs need not be co-resident), over several launches that reuse the same
counters. Each CTA:

  * writes its chunk's partials, then arrives (atomic add of 1 << 32);
  * if it was the last to arrive, takes its own share and every share marked
    abandoned in the value its add returned;
  * otherwise polls the word until all n have arrived (then takes its own
    share) or, after a bounded wait, marks its share abandoned with a
    compare-and-swap that fails once the word has changed (so once all have
    arrived), and leaves;
  * merges the shares it took, then departs; the last to depart resets the
    word and the counter for the next launch.

It checks that every share of every launch is merged exactly once, only
after all n partials are written, that the counters are zero between
launches and that nothing deadlocks. The negative tests drop one rule each
and find the failure it prevents.

A model is not the kernel: it checks the protocol's logic only.
"""
import random

import pytest

ARRIVE = 1 << 32
LOW = (1 << 32) - 1


class Violation(Exception):
    pass


def run_launches(n, slots, seed, launches=3, wait_polls=6, cas_checks_word=True, reset_by="last_departer"):
    rng = random.Random(seed)
    mem = {"word": 0, "departed": 0}
    for launch in range(launches):
        if mem["word"] != 0 or mem["departed"] != 0:
            raise Violation(f"launch {launch} starts with word {mem['word']:#x}, departed {mem['departed']}")
        written = set()
        merged = {}
        state = [{"pc": "start", "polls": 0, "mine": 0} for _ in range(n)]
        resident, waiting = [], list(range(n))
        rng.shuffle(waiting)
        done = 0

        def step(c):
            st = state[c]
            pc = st["pc"]
            if pc == "start":
                st["pc"] = "write"
            elif pc == "write":
                written.add(c)
                st["pc"] = "arrive"
            elif pc == "arrive":
                old = mem["word"]
                mem["word"] = old + ARRIVE
                st["mine"] = 1 << c
                if (old >> 32) == n - 1:
                    st["mine"] |= old & LOW
                    st["pc"] = "merge"
                    if reset_by == "last_arriver":
                        mem["word"] = 0
                else:
                    st["pc"] = "poll"
            elif pc == "poll":
                v = mem["word"]
                if (v >> 32) >= n:
                    st["pc"] = "merge"
                    return
                st["polls"] += 1
                if st["polls"] > wait_polls:
                    st["seen"] = v
                    st["pc"] = "cas"
            elif pc == "cas":
                v = st["seen"]
                if cas_checks_word:
                    if mem["word"] == v:
                        mem["word"] = v | (1 << c)
                        st["mine"] = 0
                        st["pc"] = "depart"
                    else:
                        st["pc"] = "poll"     # the word moved: look again
                else:
                    mem["word"] |= 1 << c     # a plain OR: succeeds even once all have arrived
                    st["mine"] = 0
                    st["pc"] = "depart"
            elif pc == "merge":
                m = st["mine"]
                for k in range(n):
                    if m >> k & 1:
                        if len(written) != n:
                            raise Violation(f"share {k} merged with partials {sorted(written)} of {n}")
                        merged[k] = merged.get(k, 0) + 1
                st["pc"] = "depart"
            elif pc == "depart":
                if reset_by == "last_departer":
                    d = mem["departed"]
                    mem["departed"] = d + 1
                    if d == n - 1:
                        mem["word"] = 0
                        mem["departed"] = 0
                st["pc"] = "exit"

        while done < n:
            while waiting and len(resident) < slots:
                resident.append(waiting.pop())
            c = rng.choice(resident)
            step(c)
            if state[c]["pc"] == "exit":
                resident.remove(c)
                done += 1
        for k in range(n):
            if merged.get(k, 0) != 1:
                raise Violation(f"launch {launch}: share {k} merged {merged.get(k, 0)} times")
    if mem["word"] != 0 or mem["departed"] != 0:
        raise Violation(f"counters left at word {mem['word']:#x}, departed {mem['departed']}")


def violations(cases, **kw):
    found = []
    for seed in range(cases):
        rng = random.Random(1000 + seed)
        n = rng.randint(2, 32)
        slots = rng.choice([n, n, n - 1, max(1, n // 2), 1])
        try:
            run_launches(n, slots, seed, **kw)
        except Violation as e:
            found.append((seed, n, slots, str(e)))
    return found


def test_group_protocol_merges_every_share_once():
    assert violations(600) == []


@pytest.mark.parametrize("slots", [1, 2])
def test_group_protocol_without_co_residency(slots):
    """With one or two SM slots for a group of up to 32 CTAs every early CTA
    must give its share up; the last to arrive merges them all."""
    found = []
    for seed in range(150):
        n = 2 + seed % 31
        try:
            run_launches(n, slots, seed, wait_polls=3)
        except Violation as e:
            found.append((seed, n, str(e)))
    assert found == []


def test_abandoning_without_the_compare_and_swap_loses_shares():
    """A plain OR of the abandoned bit can land after the last arrival read
    the mask: that share is merged by nobody."""
    found = violations(400, cas_checks_word=False, wait_polls=2)
    assert any("merged 0 times" in msg for *_, msg in found)


def test_reset_by_the_last_arriver_breaks_later_waiters():
    """Resetting the word when the last CTA arrives (not when the last one
    departs) lets a CTA still polling see a count of zero: it waits on, gives
    its share up into the reset word and the share is lost or carried into
    the next launch."""
    found = violations(400, reset_by="last_arriver")
    assert any("merged 0 times" in msg for *_, msg in found)
