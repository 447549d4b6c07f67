"""Model of the tcgen05 attention kernel's K/V hand-off between its persistent CTA's roles, with
mbarriers that, like the hardware's, are waited on by phase parity only.

Roles, as in csrc/attn_tc.cu: the K/V producer issues block j of an item once every group that
read block j of the previous copy has handed it back (kv_empty[j][g]); the copy lands after a
random delay (kv_full[j], waited on by the producer alone, in issue order); the producer then
passes the block to the groups that read the item (kv_ready[j][g]).  Query tiles go to the
groups (two or three) in turn across items; a group reads the blocks of its tiles in order and hands each
block back after its last tile of the item.

The model checks that every block a group reads holds its own item's data and that the run
finishes.  The same model with the earlier protocol, where the groups waited on the copy barrier
itself with the parity of their item's copy, must fail: a group that skipped an item can meet
that barrier two phases on, where a parity wait passes early.
"""
import random


class Barrier:
    """An mbarrier: `count` arrivals complete a phase; a wait on parity p passes once the phase
    with that parity has completed, i.e. while the current phase's parity differs from p."""

    def __init__(self, count=1):
        self.count, self.arrived, self.phase = count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived, self.phase = 0, self.phase + 1

    def passed(self, parity):
        return (self.phase & 1) != parity


def simulate(seed, items, per_group_ready=True, nkb_max=8, steps=200000, groups=2):
    """items: (query tiles, key blocks) per item, in the CTA's processing order."""
    rng = random.Random(seed)
    tiles = {g: [] for g in range(groups)}
    users = []
    tcount = 0
    for x, (nt, nkb) in enumerate(items):
        users.append(sum(1 << ((tcount + t) % groups) for t in range(min(nt, groups))))
        for t in range(nt):
            tiles[(tcount + t) % groups].append((x, nkb, t + groups >= nt))
        tcount += nt
    kv_full = [Barrier() for _ in range(nkb_max)]
    kv_ready = [[Barrier() for _ in range(groups)] for _ in range(nkb_max)]
    kv_empty = [[Barrier() for _ in range(groups)] for _ in range(nkb_max)]
    smem = [None] * nkb_max
    landing = []                                # (time, block, item)
    # (item, block) -> parity of kv_full for that item's copy of the block: the number of earlier
    # items that load the block, known to every role from the item list alone
    copy_parity = {(x, j): sum(1 for y in range(x) if items[y][1] > j) & 1
                   for x in range(len(items)) for j in range(items[x][1])}
    prod = dict(x=0, j=0, pend=[0] * nkb_max, e_par=[[0] * groups for _ in range(nkb_max)],
                kv_par=[0] * nkb_max, queue=[])
    grp = [dict(k=0, j=0, rpar=[0] * nkb_max, busy=0, commits=[]) for _ in range(groups)]
    for now in range(1, steps):
        for c in list(landing):
            if c[0] <= now:
                smem[c[1]] = c[2]
                kv_full[c[1]].arrive()
                landing.remove(c)
        for g in range(groups):
            for c in list(grp[g]["commits"]):
                if c[0] <= now:
                    kv_empty[c[1]][g].arrive()
                    grp[g]["commits"].remove(c)
        order = list(range(groups + 1))
        rng.shuffle(order)
        for who in order:
            if who == groups:
                # producer: issue the next copy once its block is handed back
                if prod["x"] < len(items) and len(prod["queue"]) < nkb_max:
                    x, j = prod["x"], prod["j"]
                    pend = prod["pend"][j]
                    if all(not (pend >> g) & 1 or kv_empty[j][g].passed(prod["e_par"][j][g]) for g in range(groups)):
                        for g in range(groups):
                            if (pend >> g) & 1:
                                prod["e_par"][j][g] ^= 1
                        smem[j] = ("landing", x)
                        landing.append((now + rng.randint(1, 40), j, x))
                        prod["pend"][j] = users[x]
                        if per_group_ready:
                            prod["queue"].append((j, users[x], x))
                        prod["j"] += 1
                        if prod["j"] == items[x][1]:
                            prod["x"], prod["j"] = x + 1, 0
                # producer: pass on the oldest copy once it has landed
                if prod["queue"]:
                    j, u, x = prod["queue"][0]
                    if kv_full[j].passed(prod["kv_par"][j]):
                        assert smem[j] == x
                        for g in range(groups):
                            if (u >> g) & 1:
                                kv_ready[j][g].arrive()
                        prod["kv_par"][j] ^= 1
                        prod["queue"].pop(0)
            else:
                g, st = who, grp[who]
                if st["busy"] > now or st["k"] >= len(tiles[g]):
                    continue
                x, nkb, last = tiles[g][st["k"]]
                j = st["j"]
                if per_group_ready:
                    ready = kv_ready[j][g].passed(st["rpar"][j])
                else:
                    ready = kv_full[j].passed(copy_parity[(x, j)])
                if ready:
                    if smem[j] != x:
                        return "wrong block"
                    st["busy"] = now + rng.randint(1, 30)
                    if last:
                        st["commits"].append((st["busy"] + rng.randint(0, 20), j))
                    st["j"] += 1
                    if st["j"] == nkb:
                        st["j"] = 0
                        st["k"] += 1
                        if last:
                            for jj in range(nkb):
                                st["rpar"][jj] ^= 1
        if prod["x"] >= len(items) and not prod["queue"] and all(grp[g]["k"] >= len(tiles[g]) for g in range(groups)):
            return "ok"
    return "stuck"


def _cases(n):
    for seed in range(n):
        rng = random.Random(seed)
        items = [(rng.choice([1, 1, 1, 2, 3, 4, 5, 8]), rng.randint(1, 8)) for _ in range(rng.randint(1, 12))]
        yield seed, items


import pytest


@pytest.mark.parametrize("groups", [2, 3])
def test_per_group_handoff_never_reads_a_foreign_block(groups):
    bad = [(seed, r) for seed, items in _cases(1000) for r in [simulate(seed, items, groups=groups)] if r != "ok"]
    assert not bad, bad[:5]


def test_model_finds_the_copy_barrier_aliasing():
    # the earlier protocol on the same cases: some group reads a block still landing (or waits
    # on a phase that has already gone by)
    results = [simulate(seed, items, per_group_ready=False) for seed, items in _cases(1500)]
    assert sum(r != "ok" for r in results) > 0
    assert "wrong block" in results


def simulate_descriptors(seed, blocks_per_tile, slots=4, steps=200000):
    """One group's tile descriptors.  The producer writes tile k's descriptor into slot
    k % slots once tile k - 1's queries are released (q_free: its last S product completed).  The
    issuer runs S_0, S_1, PV_0, S_2, PV_1, ..., PV_last, each S_i once the softmax has read S_{i-1}
    and each PV_m once P_m is written.  The softmax reads a tile's descriptor at its first block,
    and again when it writes the previous tile's output (during that first block, after PV of
    the previous block completed).  Returns "ok", "overwritten" (the softmax found another tile's
    descriptor in the slot) or "stuck"."""
    rng = random.Random(seed)
    n = len(blocks_per_tile)
    tile_of, last_of = [], []
    for k, nb in enumerate(blocks_per_tile):
        for j in range(nb):
            tile_of.append(k)
            last_of.append(j == nb - 1)
    total = len(tile_of)
    actions = [("S", 0)]
    for i in range(1, total):
        actions += [("S", i), ("PV", i - 1)]
    actions.append(("PV", total - 1))
    slot = [None] * slots
    published = q_free = s_done = s_read = p_written = pv_done = 0
    pending = []                       # (time, kind, block)
    a = 0                              # issuer's next action
    i_sm, phase = 0, 0                 # softmax: block, phase within it
    for now in range(1, steps):
        progress = False
        for ev in [e for e in pending if e[0] <= now]:
            pending.remove(ev)
            if ev[1] == "S":
                s_done += 1
                if last_of[ev[2]]:
                    q_free += 1
            else:
                pv_done += 1
            progress = True
        order = [0, 1, 2]
        rng.shuffle(order)
        for who in order:
            if who == 0:
                if published < n and (published == 0 or q_free >= published):
                    slot[published % slots] = published
                    published += 1
                    progress = True
            elif who == 1 and a < len(actions):
                kind, i = actions[a]
                if kind == "S" and published > tile_of[i] and (i == 0 or s_read >= i):
                    pending.append((now + rng.randint(1, 10), "S", i))
                    a += 1
                    progress = True
                elif kind == "PV" and p_written > i:
                    pending.append((now + rng.randint(1, 10), "PV", i))
                    a += 1
                    progress = True
            elif who == 2 and i_sm < total:
                k = tile_of[i_sm]
                first = i_sm == 0 or tile_of[i_sm - 1] != k
                if phase == 0 and s_done > i_sm:
                    if first and slot[k % slots] != k:
                        return "overwritten"
                    s_read = i_sm + 1
                    phase = 1
                    progress = True
                elif phase == 1 and (i_sm == 0 or pv_done >= i_sm):
                    if first and i_sm > 0 and slot[(k - 1) % slots] != k - 1:
                        return "overwritten"
                    p_written = i_sm + 1
                    i_sm, phase = i_sm + 1, 0
                    progress = True
        if i_sm == total and pv_done == total:
            return "ok" if slot[(n - 1) % slots] == n - 1 else "overwritten"
        if not progress and not pending:
            return "stuck"
    return "stuck"


@pytest.mark.parametrize("slots,expect_safe", [(4, True), (3, False)])
def test_descriptor_slots_outlive_the_output(slots, expect_safe):
    """Four slots per group (AT_DESC): a slot is rewritten only after the softmax has written the
    output of the tile it held.  Three would not be enough when a tile has one key block."""
    results = []
    for seed in range(400):
        rng = random.Random(seed)
        tiles = [rng.choice([1, 1, 1, 2, 8]) for _ in range(rng.randint(2, 20))]
        results.append(simulate_descriptors(seed, tiles, slots=slots))
    assert "stuck" not in results
    if expect_safe:
        assert all(r == "ok" for r in results)
    else:
        assert "overwritten" in results
