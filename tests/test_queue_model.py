"""A discrete-event model of the persistent kernel's expert phase, checked for
deadlock under random timings (CPU only).

The model follows the kernel's protocol: each CTA hands out work in one
in-order queue (round k: the gate/up items of entry k, then the down items of
entry k - 8; the same index formulas as the kernel); a gate/up item waits for
its ring slot's previous use to be consumed and for its chunk to land; the
last gate/up item of an entry on a CTA arrives on the entry's grid-wide
counter (a CTA without gate/up rows arrives for every entry at once); the
first down item of an entry waits for that counter to reach the grid size,
stages h and releases the entry's other down items; the producer refills a
ring slot, in entry order, once every item of its previous use is done. A run
ends when every queue is empty; a state where work remains but no event is
pending is a deadlock.
"""
import heapq
import itertools
import random

import pytest

DOWN_LAG = 8


def queue_order(U, gu_items, d_items):
    """The kernel's item order for one CTA: (is_down, entry, sub)."""
    DL = min(DOWN_LAG, U)
    n1, per2 = DL * gu_items, gu_items + d_items
    n2 = (U - DL) * per2
    out = []
    for it in range(U * (gu_items + d_items)):
        if it < n1:
            out.append((False, it // gu_items, it % gu_items))
        elif it < n1 + n2:
            r, w = divmod(it - n1, per2)
            down = w >= gu_items
            out.append((down, r if down else DL + r, w - gu_items if down else w))
        else:
            q = it - n1 - n2
            out.append((True, U - DL + q // d_items, q % d_items))
    return out


def run(G, U, gu, di, nsg, nsd, W, rng):
    """gu[b], di[b]: gate/up and down items per entry on CTA b."""
    seq = itertools.count()
    ev = []
    t = 0.0
    grid = [0] * U
    cta = []
    for b in range(G):
        c = dict(q=queue_order(U, gu[b], di[b]) if (gu[b] + di[b]) else [], head=0, free=list(range(W)), wait={},
                 lg=[0] * nsg, ld=[0] * nsd, dg=[0] * nsg, dd=[0] * nsd, hb=[0] * nsd, cnt=[0] * U,
                 ug=min(U, nsg) if gu[b] else U, ud=min(U, nsd) if di[b] else U)
        for u in range(min(U, nsg) if gu[b] else 0):
            heapq.heappush(ev, (rng.uniform(1, 3), next(seq), b, "lg", u))
        for u in range(min(U, nsd) if di[b] else 0):
            heapq.heappush(ev, (rng.uniform(1, 3), next(seq), b, "ld", u))
        if gu[b] == 0:
            for u in range(U):
                grid[u] += 1
        cta.append(c)

    def ready(b, item):
        c = cta[b]
        down, u, sub = item
        if not down:
            s, use = u % nsg, u // nsg
            return (use == 0 or c["dg"][s] >= use * gu[b]) and c["lg"][s] >= use + 1
        s, use = u % nsd, u // nsd
        if use and c["dd"][s] < use * di[b]:
            return False
        if sub == 0:
            return grid[u] >= G and c["ld"][s] >= use + 1
        return c["hb"][s] >= use + 1 and c["ld"][s] >= use + 1

    def refill(b):
        c = cta[b]
        moved = True
        while moved:
            moved = False
            if c["ug"] < U and c["dg"][c["ug"] % nsg] >= (c["ug"] // nsg) * gu[b]:
                heapq.heappush(ev, (t + rng.uniform(0.5, 3), next(seq), b, "lg", c["ug"]))
                c["ug"] += 1
                moved = True
            if c["ud"] < U and c["dd"][c["ud"] % nsd] >= (c["ud"] // nsd) * di[b]:
                heapq.heappush(ev, (t + rng.uniform(0.5, 3), next(seq), b, "ld", c["ud"]))
                c["ud"] += 1
                moved = True

    while True:
        for b, c in enumerate(cta):
            while c["free"] and c["head"] < len(c["q"]):
                c["wait"][c["free"].pop()] = c["q"][c["head"]]
                c["head"] += 1
            for w, item in list(c["wait"].items()):
                if ready(b, item):
                    del c["wait"][w]
                    down, u, sub = item
                    if down and sub == 0:  # h staged once per CTA for the entry
                        c["hb"][u % nsd] += 1
                    heapq.heappush(ev, (t + rng.uniform(0.2, 2.5), next(seq), b, "done", (w, item)))
        if not ev:
            left = [(b, c["head"], len(c["q"]), c["wait"]) for b, c in enumerate(cta)
                    if c["head"] < len(c["q"]) or c["wait"]]
            return not left, left
        t, _, b, kind, pay = heapq.heappop(ev)
        c = cta[b]
        if kind == "lg":
            c["lg"][pay % nsg] += 1
        elif kind == "ld":
            c["ld"][pay % nsd] += 1
        else:
            w, (down, u, sub) = pay
            c["free"].append(w)
            if not down:
                c["dg"][u % nsg] += 1
                c["cnt"][u] += 1
                if c["cnt"][u] == gu[b]:
                    grid[u] += 1
            else:
                c["dd"][u % nsd] += 1
        refill(b)


def test_queue_order_covers_every_item_once():
    for U in (1, 3, 8, 9, 33):
        for gi, di in ((3, 2), (1, 1), (2, 5), (0, 2), (2, 0)):
            items = queue_order(U, gi, di) if gi + di else []
            want = {(False, u, g) for u in range(U) for g in range(gi)} | {(True, u, d) for u in range(U)
                                                                             for d in range(di)}
            assert len(items) == len(want) and set(items) == want
            # every down item of an entry comes after all its gate/up items
            pos = {x: i for i, x in enumerate(items)}
            for u in range(U):
                if gi and di:
                    assert max(pos[(False, u, g)] for g in range(gi)) < min(pos[(True, u, d)] for d in range(di))


@pytest.mark.parametrize("seed", range(6))
def test_no_deadlock_under_random_timings(seed):
    rng = random.Random(seed)
    for _ in range(40):
        G = rng.randint(1, 4)
        U = rng.randint(1, 36)
        gu = [rng.choice([0, 1, 3]) for _ in range(G)]
        di = [rng.choice([0, 1, 2]) for _ in range(G)]
        nsg, nsd = rng.randint(1, 5), rng.randint(1, 5)
        W = rng.choice([1, 2, 15])
        ok, left = run(G, U, gu, di, nsg, nsd, W, rng)
        assert ok, (G, U, gu, di, nsg, nsd, W, left)
