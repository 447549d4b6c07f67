"""Model of the fused candidate pass's shared-memory ring (csrc/fm.cu), with mbarriers waited on
by phase parity only, as on the hardware.

One producer loads candidate i into stage i mod S once the stage's previous candidate (i - S)
has been released by the pair that read it; the copy lands after a random delay, possibly after
later copies.  Pair p reads candidates p, p + P, p + 2P, ...; it waits on the stage's full
barrier with the parity of candidate i's use of the stage, reads the stage and releases it.

A pair skips P - 1 of every P phases of each stage, so the parity alone is ambiguous: if the
stage's previous copy (candidate i - S) is still landing, the completed phase before it has the
same parity and the wait passes at once.  The kernel therefore tags each stage with the index of
the candidate whose copy it arms; a pair accepts a phase only when the tag is its candidate's,
and then waits once more.  The model checks that with the tag every read finds its own
candidate's rows, and that without it some read does not, even with more stages than pairs.
"""
import random

import pytest


class Barrier:
    """An mbarrier whose phases complete one by one; a wait on parity p passes while the current
    phase's parity differs from p (the phase with parity p has completed)."""

    def __init__(self):
        self.phase = 0

    def complete(self):
        self.phase += 1

    def passed(self, parity):
        return (self.phase & 1) != parity


def simulate(seed, n, stages, pairs, tagged, steps=100_000):
    rng = random.Random(seed)
    full = [Barrier() for _ in range(stages)]
    smem = [None] * stages               # candidate whose rows the stage holds (None: landing)
    tag = [-1] * stages
    released = [-1] * stages             # last candidate read out of the stage
    landing = []                         # (time, stage, candidate)
    nxt = 0                              # producer's next candidate
    cur = list(range(pairs))             # each pair's current candidate
    state = ["wait"] * pairs             # "wait" -> ("check" ->) "read" -> "busy"
    busy_until = [0] * pairs
    for now in range(1, steps):
        # copies complete out of order; a stage's copy completes its next phase
        for c in sorted((c for c in landing if c[0] <= now), key=lambda c: c[0]):
            landing.remove(c)
            smem[c[1]] = c[2]
            full[c[1]].complete()
        # producer: one copy per step, in candidate order, once the stage is free
        if nxt < n:
            st = nxt % stages
            if nxt < stages or released[st] == nxt - stages:
                tag[st] = nxt
                smem[st] = None
                # mostly quick copies, now and then a very late one
                delay = rng.randint(1, 6) if rng.random() < 0.9 else rng.randint(20, 120)
                landing.append((now + delay, st, nxt))
                nxt += 1
        order = list(range(pairs))
        rng.shuffle(order)
        for p in order:
            i = cur[p]
            if i >= n or busy_until[p] > now:
                continue
            st, par = i % stages, (i // stages) & 1
            if state[p] == "wait":
                if full[st].passed(par):
                    state[p] = "check" if tagged else "read"
            elif state[p] == "check":
                # the tag names the candidate whose copy the stage was last armed for
                if tag[st] == i and full[st].passed(par):
                    state[p] = "read"
                elif tag[st] != i:
                    state[p] = "wait"
            if state[p] == "read":
                if smem[st] != i:
                    return "wrong rows"
                released[st] = i
                busy_until[p] = now + rng.randint(1, 8)
                cur[p] = i + pairs
                state[p] = "wait"
        if nxt >= n and not landing and all(c >= n for c in cur):
            return "ok"
    return "stuck"


def _cases(k):
    for seed in range(k):
        yield seed, random.Random(seed).randint(20, 120)


@pytest.mark.parametrize("stages,pairs", [(12, 7), (8, 7), (7, 7)])
def test_tagged_ring_reads_only_its_own_rows(stages, pairs):
    bad = [(s, r) for s, n in _cases(400) for r in [simulate(s, n, stages, pairs, tagged=True)] if r != "ok"]
    assert not bad, bad[:5]


@pytest.mark.parametrize("stages,pairs", [(12, 7), (6, 7)])
def test_parity_alone_reads_stale_rows(stages, pairs):
    # the protocol before the tag: a late copy lets a pair's parity wait pass one phase early,
    # with more stages than pairs too
    results = [simulate(s, n, stages, pairs, tagged=False) for s, n in _cases(400)]
    assert "wrong rows" in results
